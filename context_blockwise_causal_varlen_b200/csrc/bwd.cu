// Block backward on tcgen05, fed the MERGED softmax statistics.
//
// NeMo AutoModel, zigzag_ring_attention: _block_backward and
// zigzag_ring_flash_attn_varlen_backward ("each block's flash backward is fed the
// FINAL merged out/lse"); ulysses_attention._block0_backward.  With
// P = exp(scale q k^T - lse) over a block's visible pairs and Delta = rowsum(dO * O):
//   dV += P^T dO,  dP = dO V^T,  dS = P * (dP - Delta),  dQ += scale dS K,  dK += scale dS^T Q.
//
// One CTA owns a 128-key tile of one kv head and streams 64-row q tiles from every
// segment (ring block) that sees it, for every q head of its GQA group, so dK and dV
// accumulate in TMEM across all blocks and are written once (the ring's "K/V grads
// travel back to their owner" becomes accumulation in place).  dQ^T = K^T dS^T is
// formed per q tile in TMEM and added to an fp32 dq accumulator with a TMA bulk
// reduce-add.
//
// Warps: 0 TMA producer (q, dO, lse*log2e and Delta rows of a 3-stage ring),
// 1 UMMA issuer (+ TMEM owner; the whole warp runs the loop, one elected lane issues), 2-9 P / dS in two warpgroups that split the 64
// q columns (one key row per thread) and then the dV / dK epilogue, 10-13 dQ readout.
// TMEM columns: S^T [0,64), dP^T [64,128), dQ^T [128,192), P^T [192,256) (two buffers of 32 columns,
// bf16 pairs), dV [256,256+D), dK [384,384+D).  P^T goes from the softmax warps' registers straight
// into TMEM as the A operand of dV = P^T dO: a store to shared memory would have to complete before
// the hand-off to the UMMA issuer, and those stores, not the UMMAs' operand reads, are what the
// shared memory spends its time on.  dS^T still goes to shared memory: it is also dQ^T's B operand.
#include "kernels.h"
#include "ptx.cuh"

namespace cbv {

namespace {

constexpr int BN = 128;  // keys per CTA
constexpr int BM = 64;   // q rows per streamed tile
constexpr int kThreads = 448;
constexpr int NS = 3;     // q / dO / row stages
constexpr int kRowPairs = BM + 2;  // {lse, Delta} box: 66 pairs from a 16-byte aligned start
constexpr int kRowSlot = 160;      // floats per stage: 640 bytes keeps every TMA destination 128-byte aligned
constexpr int kDQRows = 16;      // q rows per dQ bulk reduce (four per q tile)

struct QTile {
  int32_t q_row;   // first q row
  int32_t qpos0;   // its position
  int32_t nvalid;  // valid rows
  int32_t head;    // q head
  int32_t causal;
  int32_t need_mask;
};

struct QIter {
  int32_t hs = 0, si = 0, j = 0, jn = 0;
  Seg seg;
};

// Enumerates the q tiles (over the GQA group's q heads and all segments) that see
// at least one key of the tile.  Every role runs its own copy.
__device__ __forceinline__ bool next_qtile(const BwdParams& p, const TileTask& t, int kvh, QIter& it, QTile& r) {
  // key positions span [kp0, kp1]: with a second range, its last key (it lies after the first)
  const int32_t kp0 = t.pos0, kp1 = t.split1 ? max(t.pos0 + t.rows, t.pos1 + t.rows1) - 1 : t.pos0 + t.rows - 1;
  const int32_t W = p.window;
  while (true) {
    if (it.hs >= p.heads_per_kv) return false;  // exhausted (and stays so when called again)
    if (it.j >= it.jn) {
      if (it.si >= t.nseg) {
        it.hs++;
        it.si = 0;
        if (it.hs >= p.heads_per_kv) return false;
      }
      if (t.nseg == 0) return false;
      it.seg = p.segs[t.seg0 + it.si];
      it.si++;
      // a tile of two key ranges tests causality on every segment: a segment that lies wholly
      // after one range's keys can still precede the other's (the test is a no-op elsewhere)
      const bool cz = (it.seg.flags & kSegCausal) || W > 0 || t.split1;
      int32_t cmin = 0, cmax = it.seg.rows - 1;
      if (cz) cmin = max(cmin, kp0 - it.seg.pos0);
      if (W > 0) cmax = min(cmax, kp1 + W - 1 - it.seg.pos0);
      if (cmax < cmin) {
        it.j = it.jn = 0;
        continue;
      }
      it.j = cmin / BM;
      it.jn = cmax / BM + 1;
    }
    const int32_t j = it.j++;
    const int32_t c0 = j * BM;
    r.nvalid = min(BM, it.seg.rows - c0);
    r.q_row = it.seg.row0 + c0;
    r.qpos0 = it.seg.pos0 + c0;
    r.head = kvh * p.heads_per_kv + it.hs;
    r.causal = (it.seg.flags & kSegCausal) || t.split1;
    const bool cz = r.causal || W > 0;
    const int32_t qa = r.qpos0, qb = r.qpos0 + r.nvalid - 1;
    const bool all_vis = (r.nvalid == BM) && (t.rows == BN) && (!cz || qa >= kp1) && (W <= 0 || qb - kp0 < W);
    r.need_mask = !all_vis;
    return true;
  }
}

template <int D>
struct BwdSmem {
  static constexpr uint32_t kKV = BN * D * 2;   // K or V tile (128 x D)
  static constexpr uint32_t kQT = BM * D * 2;   // a q / dO tile (64 x D)
  static constexpr uint32_t kPT = BN * BM * 2;  // dS^T (128 x 64)
  static constexpr uint32_t kRowBytes = kRowPairs * 8;  // bytes one row box delivers
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kKV;
  static constexpr uint32_t kQ = kV + kKV;            // NS stages
  static constexpr uint32_t kDO = kQ + NS * kQT;      // NS stages
  static constexpr uint32_t kDSt = kDO + NS * kQT;       // dS^T, two buffers (q tile j uses j & 1)
  static constexpr uint32_t kDSt1 = kDSt + kPT;
  static constexpr uint32_t kDQBuf = kDQRows * D * 4;     // fp32 staging buffer: 4 warps x [16][D/4]
  static constexpr uint32_t kDQ = kDSt1 + kPT;            // two staging buffers
  static constexpr uint32_t kRow = kDQ + 2 * kDQBuf;      // per stage: lse*log2e and Delta slots
  static constexpr uint32_t kBars = kRow + NS * kRowSlot * 4;
  static constexpr uint32_t kEnd = kBars + 256;
  static constexpr uint32_t kDynamic = (kEnd + 1024) < 120 * 1024 ? 120 * 1024 : (kEnd + 1024);
  static_assert(kDynamic <= 232448, "shared memory budget");
};

enum BBar {
  bKVFull = 0,
  bQFull = 1,    // +stage (NS)
  bQEmpty = 4,   // +stage (NS)
  bSFull = 7,
  bSFree = 8,
  bPFull = 9,    // +buffer (2): P^T (TMEM) and dS^T (shared memory) written
  bPtFree = 11,  // +buffer (2): the UMMAs that read P^T / dS^T buffer b have completed
  bDQFull = 13,
  bDQFree = 14,
  bUnused15 = 15,
  bAccDone = 16,
  bBNum = 17
};


template <int D>
__global__ void __launch_bounds__(kThreads, 1) bwd_kernel(const __grid_constant__ BwdParams p) {
  using L = BwdSmem<D>;
  constexpr int KH = D / 64;  // 64-column halves
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align_smem_1024(smem_raw);
  uint8_t* sK = sm + L::kK;
  uint8_t* sV = sm + L::kV;
  uint8_t* sQ = sm + L::kQ;
  uint8_t* sDO = sm + L::kDO;
  uint8_t* sDSt = sm + L::kDSt;
  float* sDQ = reinterpret_cast<float*>(sm + L::kDQ);
  float* sRow = reinterpret_cast<float*>(sm + L::kRow);  // [stage][66 pairs {lse*log2e, Delta}]
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + bBNum);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const TileTask t = p.tasks[blockIdx.x];
  const int kvh = t.head;

  if (threadIdx.x == 0) {
    mbar_init(&bar[bKVFull], 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar[bQFull + s], 1);
      mbar_init(&bar[bQEmpty + s], 1);
    }
    mbar_init(&bar[bDQFull], 1);
    mbar_init(&bar[bDQFree], 4);
    mbar_init(&bar[bSFull], 1);
    mbar_init(&bar[bSFree], 8);
    mbar_init(&bar[bPFull], 8);
    mbar_init(&bar[bPFull + 1], 8);
    mbar_init(&bar[bPtFree], 1);
    mbar_init(&bar[bPtFree + 1], 1);
    mbar_init(&bar[bAccDone], 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tDP = tmem + 64, tDQ = tmem + 128, tPt = tmem + 192, tDV = tmem + 256, tDK = tmem + 384;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_q);
      if (p.prefetch_ahead > 0 && (int)blockIdx.x + p.prefetch_ahead < p.num_tasks) {
        // warm L2 with the keys and values of the task that will likely start on an SM when this
        // wave ends, so its start waits on L2 rather than on HBM
        const TileTask nx = p.tasks[blockIdx.x + p.prefetch_ahead];
        for (int h = 0; h < KH; ++h) {
          tma_prefetch_l2_3d(&p.tm_k, h * 64, nx.head, nx.row0);
          tma_prefetch_l2_3d(&p.tm_v, h * 64, nx.head, nx.row0);
          if (nx.split1) {
            tma_prefetch_l2_3d(&p.tm_k, h * 64, nx.head, nx.row1);
            tma_prefetch_l2_3d(&p.tm_v, h * 64, nx.head, nx.row1);
          }
        }
      }
      mbar_arrive_expect_tx(&bar[bKVFull], 2 * L::kKV);
      for (int h = 0; h < KH; ++h) {
        if (!t.split1) {
          int32_t kr = t.row0;
          CBV_CHECK_RANGE(kr, 0, p.kv_rows, p.status, kDevBoundsKV);
          tma_load_3d(sK + h * 16384, &p.tm_k, &bar[bKVFull], h * 64, kvh, kr);
          tma_load_3d(sV + h * 16384, &p.tm_v, &bar[bKVFull], h * 64, kvh, kr);
        } else {
          // two key ranges: 8-row pieces (1 KB of the 128B-swizzled tile each, so the swizzle
          // pattern stays aligned); every tile row is loaded, from one range or the other
          for (int g = 0; g < BN / 8; ++g) {
            int32_t row = g * 8 < t.split1 ? t.row0 + g * 8 : t.row1 + (g * 8 - t.split1);
#ifdef CBV_DEBUG
            // pieces past a range's valid keys may start past the tensor (the copy reads zeros there)
            if (g * 8 < t.split1 ? g * 8 < t.rows : g * 8 - t.split1 < t.rows1)
              CBV_CHECK_RANGE(row, 0, p.kv_rows, p.status, kDevBoundsKV);
#endif
            tma_load_3d(sK + h * 16384 + g * 1024, &p.tm_k8, &bar[bKVFull], h * 64, kvh, row);
            tma_load_3d(sV + h * 16384 + g * 1024, &p.tm_v8, &bar[bKVFull], h * 64, kvh, row);
          }
        }
      }
    }
    if (lane == 0) {
      QIter it;
      QTile r;
      int j = 0;
      while (next_qtile(p, t, kvh, it, r)) {
        const int st = j % NS;
        if (!mbar_wait(&bar[bQEmpty + st], ((j / NS) & 1) ^ 1, p.status, kDevTimeoutTmaEmpty)) break;
        uint64_t* full = &bar[bQFull + st];
        mbar_arrive_expect_tx(full, 2 * L::kQT + L::kRowBytes);
        CBV_CHECK_RANGE(r.q_row, 0, p.q_rows, p.status, kDevBoundsQ);
        for (int h = 0; h < KH; ++h) {
          tma_load_3d(sQ + st * L::kQT + h * 8192, &p.tm_q, full, h * 64, r.head, r.q_row);
          tma_load_3d(sDO + st * L::kQT + h * 8192, &p.tm_do, full, h * 64, r.head, r.q_row);
        }
        // pairs from an even q row (a 16-byte aligned start); the softmax indexes from q_row & 1
        tma_load_2d(sRow + st * kRowSlot, &p.tm_rows, full, 2 * (r.q_row & ~1), r.head);
        ++j;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ UMMA issuer (whole warp, one lane issues)
    {
      constexpr uint32_t id_st = idesc_bf16(BN, BM, false, false);   // S^T, dP^T: 128 x 64, K = D
      constexpr uint32_t id_kv = idesc_bf16(BN, D, false, true);     // dV, dK: 128 x D, K = 64
      constexpr uint32_t id_dq = idesc_bf16(D, BM, true, true);      // dQ^T: D x 64, K = 128
      // base descriptors, built once; per-instruction offsets are compile-time constants
      const uint64_t dK_k = sdesc_sw128(smem_u32(sK), 16, 1024);        // K as K-major A (S^T)
      const uint64_t dK_mn = sdesc_sw128(smem_u32(sK), 16384, 1024);    // K^T as MN-major A (dQ^T)
      const uint64_t dV_k = sdesc_sw128(smem_u32(sV), 16, 1024);        // V as K-major A (dP^T)
      // dS^T buffer b of 2 (q tile j uses buffer j & 1; P^T's buffer b is TMEM columns tPt + 32 b)
      const uint64_t dDSt[2] = {sdesc_sw128(smem_u32(sDSt), 16, 1024),     // dS^T, K-major A (dK)
                                sdesc_sw128(smem_u32(sm + L::kDSt1), 16, 1024)};
      const uint64_t dDSt_mn[2] = {sdesc_sw128(smem_u32(sDSt), 16384, 1024),  // dS^T, MN-major B (dQ^T)
                                   sdesc_sw128(smem_u32(sm + L::kDSt1), 16384, 1024)};
      // stage s of q / dO sits s * kQT bytes after stage 0
      const uint64_t dQ_k = sdesc_sw128(smem_u32(sQ), 16, 1024);       // q as K-major B (S^T)
      const uint64_t dO_k = sdesc_sw128(smem_u32(sDO), 16, 1024);      // dO as K-major B (dP^T)
      const uint64_t dQ_mn = sdesc_sw128(smem_u32(sQ), 8192, 1024);    // q as MN-major B (dK)
      const uint64_t dO_mn = sdesc_sw128(smem_u32(sDO), 8192, 1024);   // dO as MN-major B (dV)
      bool ok = mbar_wait_warp(&bar[bKVFull], 0, p.status, kDevTimeoutMma);
      tc_fence_after();
      auto issue_sdp = [&](int j) -> bool {
        const int st = j % NS;
        if (!mbar_wait_warp(&bar[bQFull + st], (j / NS) & 1, p.status, kDevTimeoutMma)) return false;
        if (!mbar_wait_warp(&bar[bSFree], (j & 1) ^ 1, p.status, kDevTimeoutMma)) return false;
        tc_fence_after();
        const uint64_t bq = sdesc_add(dQ_k, st * L::kQT), bo = sdesc_add(dO_k, st * L::kQT);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ao = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t bb = (kk >> 2) * 8192 + (kk & 3) * 32;
          umma_bf16_ss(tS, sdesc_add(dK_k, ao), sdesc_add(bq, bb), id_st, kk > 0);
          umma_bf16_ss(tDP, sdesc_add(dV_k, ao), sdesc_add(bo, bb), id_st, kk > 0);
        }
        umma_commit(&bar[bSFull]);
        return true;
      };
      QIter it;
      QTile r;
      int n = 0;
      {
        QIter c2;
        QTile r2;
        while (next_qtile(p, t, kvh, c2, r2)) ++n;
      }
      if (ok && n > 0) ok = issue_sdp(0);
      for (int j = 0; ok && j < n; ++j) {
        const int st = j % NS;
        if (j + 1 < n && !(ok = issue_sdp(j + 1))) break;
        // one PFull per P^T / dS^T buffer: a fast softmax warp may finish tile j + 1 before a slow
        // one has finished tile j, and their arrivals must not complete the same phase
        const int pb = j & 1;
        if (!mbar_wait_warp(&bar[bPFull + pb], (j >> 1) & 1, p.status, kDevTimeoutMma)) { ok = false; break; }
        tc_fence_after();
        const uint64_t omn = sdesc_add(dO_mn, st * L::kQT), qmn = sdesc_add(dQ_mn, st * L::kQT);
        const uint64_t ads = pb ? dDSt[1] : dDSt[0];
        const uint64_t bds = pb ? dDSt_mn[1] : dDSt_mn[0];
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk) {
          const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
          umma_bf16_ts(tDV, tPt + pb * 32 + kk * 8, sdesc_add(omn, kk * 2048), id_kv, acc);
          umma_bf16_ss(tDK, sdesc_add(ads, kk * 32), sdesc_add(qmn, kk * 2048), id_kv, acc);
        }
        if (!mbar_wait_warp(&bar[bDQFree], (j & 1) ^ 1, p.status, kDevTimeoutMma)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tdq = tDQ;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_bf16_ss(tdq, sdesc_add(dK_mn, kk * 2048), sdesc_add(bds, kk * 2048), id_dq, kk > 0 ? 1u : 0u);
        umma_commit(&bar[bQEmpty + st]);
        umma_commit(&bar[bPtFree + pb]);
        umma_commit(&bar[bDQFull]);
      }
      (void)it;
      (void)r;
      if (n > 0) umma_commit(&bar[bAccDone]);
      else if (lane == 0) mbar_arrive(&bar[bAccDone]);
    }
  } else if (warp < 10) {
    // ------------------------------------------------------------------ P / dS (thread = key row)
    // warpgroup wg handles q columns [32 wg, 32 wg + 32) of every tile
    const int wg = (warp - 2) >> 2;
    const int c0 = wg * 32;
    const int quarter = warp & 3;
    const int krow = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const bool second = t.split1 && krow >= t.split1;  // this key row belongs to the second range
    const int32_t kpos = second ? t.pos1 + (krow - t.split1) : t.pos0 + krow;
    bool kvalid = second ? krow - t.split1 < t.rows1 : krow < t.rows;
    const int32_t kglobal = second ? t.row1 + (krow - t.split1) : t.row0 + krow;
#ifdef CBV_DEBUG
    if (kvalid && (kglobal < 0 || kglobal >= p.kv_rows)) {
      atomicCAS(p.status, 0, kDevBoundsOut);
      kvalid = false;
    }
#endif
    const int32_t W = p.window;
    const float sl2 = p.scale_log2;
    const uint32_t ds_buf[2] = {smem_u32(sDSt), smem_u32(sm + L::kDSt1)};
    bool ok = true;
    QIter it;
    QTile r;
    int j = 0;
    while (ok && next_qtile(p, t, kvh, it, r)) {
      const int st = j % NS;
      if (!mbar_wait_warp(&bar[bQFull + st], (j / NS) & 1, p.status, kDevTimeoutSoftmax)) { ok = false; break; }
      if (!mbar_wait_warp(&bar[bSFull], j & 1, p.status, kDevTimeoutSoftmax)) { ok = false; break; }
      tc_fence_after();
      const float2* lrow = reinterpret_cast<const float2*>(sRow + st * kRowSlot) + (r.q_row & 1) + c0;
      uint32_t pp[16], pd[16];
      {
        uint32_t s[32], dp[32];
        tmem_ld32(tS + lane_base + c0, s);
        tmem_ld32(tDP + lane_base + c0, dp);
        tmem_ld_wait();
        // S^T / dP^T are in registers: release the TMEM buffers so the next tile's
        // S^T and dP^T can be computed while this one is being turned into P and dS
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[bSFree]);
        bool skip = false;  // no row of this warp sees any of its 32 q columns
        if (r.need_mask) {
          // this key row sees the q columns [lo, hi] (positions are linear in the column).  The
          // others get a score of -inf and then the same arithmetic as visible ones: every
          // {lse * log2e, Delta} the row box delivers is finite (rows with no visible key store 0,
          // pad rows are zero, past the tensor the box reads zeros), so P and dS come out 0.
          // A warp whose rows all see every column skips the mask, one whose rows see none skips
          // the arithmetic too (its P and dS are zeros).
          int32_t hi = kvalid ? r.nvalid - 1 : -1, lo = 0;
          if (r.causal || W > 0) lo = max(lo, kpos - r.qpos0);
          if (W > 0) hi = min(hi, kpos + W - 1 - r.qpos0);
          lo -= c0;
          hi -= c0;
          skip = __all_sync(0xffffffffu, hi < 0 || lo > 31 || hi < lo);
          if (!skip && !__all_sync(0xffffffffu, lo <= 0 && hi >= 31)) {
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (c < lo || c > hi) s[c] = __float_as_uint(-INFINITY);
          }
        }
        if (skip) {
#pragma unroll
          for (int c = 0; c < 16; ++c) pp[c] = pd[c] = 0u;
        } else {
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float2 r0 = lrow[c], r1 = lrow[c + 1];
            const float p0 = ex2_approx(fmaf(__uint_as_float(s[c]), sl2, -r0.x));
            const float p1 = ex2_approx(fmaf(__uint_as_float(s[c + 1]), sl2, -r1.x));
            pp[c / 2] = pack_bf16x2(p0, p1);
            pd[c / 2] = pack_bf16x2(p0 * (__uint_as_float(dp[c]) - r0.y), p1 * (__uint_as_float(dp[c + 1]) - r1.y));
          }
        }
      }
      // buffer j & 1 was last read by the UMMAs of q tile j - 2
      const int pb = j & 1;
      if (j >= 2 && !mbar_wait_warp(&bar[bPtFree + pb], ((j >> 1) - 1) & 1, p.status, kDevTimeoutSoftmax)) {
        ok = false;
        break;
      }
      // P^T: this key row's 32 q columns as 16 bf16 pairs, columns [c0 / 2, c0 / 2 + 16) of the buffer
      tmem_st16(tPt + lane_base + pb * 32 + (c0 >> 1), pp);
      const uint32_t ds_row = pb ? ds_buf[1] : ds_buf[0];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch)
        st_shared_v4(ds_row + sw128_offset(krow, (c0 >> 3) + ch), pd[ch * 4], pd[ch * 4 + 1], pd[ch * 4 + 2],
                     pd[ch * 4 + 3]);
      tmem_st_wait();
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[bPFull + pb]);
      ++j;
    }
    // ---------------------------------------------------------------- dK / dV epilogue
    if (ok && mbar_wait_warp(&bar[bAccDone], 0, p.status, kDevTimeoutEpilogue)) {
      tc_fence_after();
      const bool any = j > 0;
      const int which = wg;  // warpgroup 0: dV, warpgroup 1: dK
      const uint32_t tsrc = (which == 0 ? tDV : tDK) + lane_base;
      const float mul = which == 0 ? 1.f : p.scale;
      void* dst_base = which == 0 ? p.dv : p.dk;
      if (!p.dkv_accumulate) {
        // bf16 out through shared memory, so that the global stores are whole rows: each warp
        // stages its 32 key rows in the K / V tiles (every MMA that read them has completed), then
        // consecutive lanes store consecutive 16-byte pieces of a row
        constexpr int UPR = D / 8;  // 16-byte units per row
        const uint32_t stg = smem_u32(sm + L::kK) + (uint32_t)(wg * 4 + quarter) * (32 * D * 2);
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          tmem_ld32(tsrc + c, o);
          tmem_ld_wait();
#pragma unroll
          for (int u4 = 0; u4 < 4; ++u4) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = any ? __uint_as_float(o[u4 * 8 + e]) * mul : 0.f;
            const int unit = c / 8 + u4;
            st_shared_v4(stg + lane * (D * 2) + ((unit ^ (lane & (UPR - 1))) << 4), pack_bf16x2(x[0], x[1]),
                         pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
          }
        }
        __syncwarp();
        constexpr int RPI = 32 / UPR;  // rows per store instruction
        const int sub = lane / UPR, unit = lane % UPR;
#pragma unroll
        for (int i = 0; i < 32 / RPI; ++i) {
          const int lr = i * RPI + sub;
          const int kr = quarter * 32 + lr;
          const bool sec = t.split1 && kr >= t.split1;
          bool valid = sec ? kr - t.split1 < t.rows1 : kr < t.rows;
          uint32_t v4[4];
          ld_shared_v4(stg + lr * (D * 2) + ((unit ^ (lr & (UPR - 1))) << 4), v4);
          const int64_t kg = sec ? (int64_t)t.row1 + (kr - t.split1) : (int64_t)t.row0 + kr;
#ifdef CBV_DEBUG
          if (valid && (kg < 0 || kg >= p.kv_rows)) {
            atomicCAS(p.status, 0, kDevBoundsOut);
            valid = false;
          }
#endif
          if (valid) {
            __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(dst_base) + kg * p.dkv_stride_t +
                                 (int64_t)kvh * p.dkv_stride_h + unit * 8;
            *reinterpret_cast<uint4*>(dst) = make_uint4(v4[0], v4[1], v4[2], v4[3]);
          }
        }
      } else {
        const int64_t off = (int64_t)kglobal * p.dkv_stride_t + (int64_t)kvh * p.dkv_stride_h;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          tmem_ld32(tsrc + c, o);
          tmem_ld_wait();
          if (!kvalid || !any) continue;
          float* dst = reinterpret_cast<float*>(dst_base) + off + c;
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            float4 a = *reinterpret_cast<float4*>(dst + e);
            a.x += __uint_as_float(o[e]) * mul;
            a.y += __uint_as_float(o[e + 1]) * mul;
            a.z += __uint_as_float(o[e + 2]) * mul;
            a.w += __uint_as_float(o[e + 3]) * mul;
            *reinterpret_cast<float4*>(dst + e) = a;
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ dQ readout (thread = head-dim row)
    // Each warp owns D/4 head-dim rows and adds its [16 x D/4] slices (four per q tile)
    // with its own bulk reduces, so the four warps never wait on one another.
    const int quarter = warp & 3;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    constexpr int DW = D / 4;  // head-dim rows per warp
    // M = 128: lane l of quarter q holds d = 32q + l; M = 64: lanes 0-15 of quarter q hold d = 16q + l
    const bool dvalid = lane < DW;
    // two staging buffers per warp, used in turn, so the reduce in flight never blocks the next slice
    float* region0 = sDQ + quarter * (kDQRows * DW);
    QIter it;
    QTile r;
    int j = 0;
    while (next_qtile(p, t, kvh, it, r)) {
      if (!mbar_wait_warp(&bar[bDQFull], j & 1, p.status, kDevTimeoutEpilogue)) break;
      tc_fence_after();
      uint32_t v[BM];
      tmem_ld32(tDQ + lane_base, v);
      tmem_ld32(tDQ + lane_base + 32, v + 32);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[bDQFree]);
      if (p.dq_fixed == nullptr) {
#pragma unroll
        for (int pc = 0; pc < BM / kDQRows; ++pc) {
          float* region = region0 + (pc & 1) * (L::kDQBuf / 4);
          if (lane == 0) bulk_wait_group_read<1>();  // the reduce that last used this buffer has read it
          __syncwarp();
          if (dvalid) {
#pragma unroll
            for (int c = 0; c < kDQRows; ++c) region[c * DW + lane] = __uint_as_float(v[pc * kDQRows + c]) * p.scale;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_reduce_add_3d(&p.tm_dq, region, quarter * DW, r.head, r.q_row + pc * kDQRows);
            bulk_commit_group();
          }
        }
      } else {
        // Deterministic: 8-row slices of 64-bit fixed point (units of 2^-32) in the same buffers,
        // each added by one integer bulk reduce (the accumulator keeps a warp's rows contiguous).
        // Rows past the tile's valid rows hold exact zeros, as in the fp32 path.
        constexpr int kFixRows = kDQRows / 2;
        unsigned long long* fregion0 = reinterpret_cast<unsigned long long*>(region0);
        const float fscale = p.scale * 4294967296.f;
#pragma unroll
        for (int pc = 0; pc < BM / kFixRows; ++pc) {
          unsigned long long* region = fregion0 + (pc & 1) * (L::kDQBuf / 8);
          if (lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
          if (dvalid) {
#pragma unroll
            for (int c = 0; c < kFixRows; ++c)
              region[c * DW + lane] =
                  (unsigned long long)__float2ll_rn(__uint_as_float(v[pc * kFixRows + c]) * fscale);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (pc * kFixRows < r.nvalid)
              bulk_reduce_add_u64(p.dq_fixed + fixed_index(r.q_row + pc * kFixRows, r.head, quarter * DW,
                                                           p.dq_fixed_tpad, D),
                                  region, kFixRows * DW * 8);
            bulk_commit_group();
          }
        }
      }
      ++j;
    }
    // the staging buffers must outlive only the reads of the last reduces; their additions into the
    // accumulator are complete when the grid is, before any later kernel on the stream reads it
    if (lane == 0) bulk_wait_group_read<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int D>
int launch_bwd_t(const BwdParams& p, int grid, cudaStream_t stream) {
  auto kern = bwd_kernel<D>;
  const uint32_t smem = BwdSmem<D>::kDynamic;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return (int)e;
  if (const int ev = kernel_event_start(stream)) return ev;
  kern<<<grid, kThreads, smem, stream>>>(p);
  const int rc = launched();
  if (rc) return rc;
  return kernel_event_stop(stream);
}

}  // namespace

int launch_bwd(const BwdParams& p, int head_dim, int grid, cudaStream_t stream) {
  if (grid <= 0) return 0;
  if (head_dim == 128) return launch_bwd_t<128>(p, grid, stream);
  if (head_dim == 64) return launch_bwd_t<64>(p, grid, stream);
  return (int)cudaErrorInvalidValue;
}

}  // namespace cbv
