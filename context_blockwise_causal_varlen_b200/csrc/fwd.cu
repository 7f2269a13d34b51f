// Block forward on tcgen05: flash-style attention of one 128-row q tile against a
// list of k/v segments, returning (out, lse) or merging into a running pair.
//
// This is the per-block kernel of the NeMo AutoModel zig-zag ring page
// (_block_forward: one flash varlen forward block) and of the KV-parallel
// segmented prefill (NKI attention_kv_parallel_segmented_cte: per-shard segment
// loop with online softmax).  Consecutive segments belonging to different ring
// blocks (or shards) are combined by the online-softmax log-sum-exp identity
// (update_out_and_lse) applied in place to the TMEM accumulator; with
// out_mode = kOutMerge the epilogue applies the same identity to a running
// (out, lse) pair held in HBM, so no separate merge pass is needed.
//
// CTA = 6 warps: warp 0 issues TMA loads, warp 1 issues UMMAs (and owns TMEM),
// warps 2-5 run the softmax / correction / epilogue for one row each.
// TMEM columns: S double buffer [0,128) and [128,256), O accumulator [256, 256+D).
#include "kernels.h"
#include "ptx.cuh"

namespace cbv {

namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int kThreads = 192;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: keep a stale max while it is within 2^8

struct TileRef {
  int32_t k_row;    // first row (non-paged: tensor row; paged: shard-local token)
  int32_t kpos0;    // position of column 0 (paged: position of the tile's first token)
  int32_t nvalid;   // valid columns
  int32_t causal;
  int32_t need_mask;
  int32_t shard;
};

struct TileIter {
  int32_t si = 0, j = 0, jn = 0;
  Seg seg;
};

__device__ __forceinline__ int32_t kvp_pos_dev(const FwdParams& p, int32_t shard, int32_t t) {
  if (p.kv_mode == kKvRoundRobin)
    return ((t / p.block_size) * p.shards + shard) * p.block_size + t % p.block_size;
  return shard * p.n_local + t;
}

// Enumerates the k tiles of a task that at least one row of the q tile can see.
// Every role runs its own copy and sees the same sequence.
template <bool PAGED>
__device__ __forceinline__ bool next_tile(const FwdParams& p, const TileTask& t, TileIter& it, TileRef& r) {
  const int32_t qp0 = t.pos0, qp1 = t.pos0 + t.rows - 1;
  const int32_t W = p.window;
  while (true) {
    if (it.j >= it.jn) {
      if (it.si >= t.nseg) return false;
      it.seg = p.segs[t.seg0 + it.si];
      it.si++;
      const int32_t rows = it.seg.rows;
      if (!PAGED) {
        const bool cz = (it.seg.flags & kSegCausal) || W > 0;
        int32_t cmax = rows - 1, cmin = 0;
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
        it.jn = (rows + BN - 1) / BN;
      }
    }
    const int32_t j = it.j++;
    const int32_t c0 = j * BN;
    r.nvalid = min(BN, it.seg.rows - c0);
    r.k_row = it.seg.row0 + c0;
    r.causal = it.seg.flags & kSegCausal;
    int32_t kmin, kmax;
    if (!PAGED) {
      r.shard = 0;
      r.kpos0 = it.seg.pos0 + c0;
      kmin = r.kpos0;
      kmax = r.kpos0 + r.nvalid - 1;
    } else {
      r.shard = it.seg.flags >> kSegShardShift;
      kmin = kvp_pos_dev(p, r.shard, r.k_row);
      kmax = kvp_pos_dev(p, r.shard, r.k_row + r.nvalid - 1);
      r.kpos0 = kmin;
      if (kmin > qp1) continue;
      if (W > 0 && kmax < qp0 - W + 1) continue;
    }
    const bool cz = r.causal || W > 0;
    const bool all_vis = (r.nvalid == BN) && (!cz || kmax <= qp0) && (W <= 0 || qp1 - kmin < W);
    r.need_mask = !all_vis;
    return true;
  }
}

template <int D>
struct FwdSmem {
  static constexpr uint32_t kTileBytes = BM * D * 2;  // a 128 x D bf16 tile
  static constexpr uint32_t kPBytes = BM * BN * 2;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kTileBytes;
  static constexpr uint32_t kV = kK + 2 * kTileBytes;
  static constexpr uint32_t kP = kV + 2 * kTileBytes;
  static constexpr uint32_t kBars = kP + kPBytes;
  static constexpr uint32_t kEnd = kBars + 256;
  // one CTA per SM (TMEM: 512 columns per CTA)
  static constexpr uint32_t kDynamic = (kEnd + 1024) < 120 * 1024 ? 120 * 1024 : (kEnd + 1024);
};

enum Bar {
  bQFull = 0,
  bKFull = 1,   // +stage
  bVFull = 3,   // +stage
  bKEmpty = 5,  // +stage
  bVEmpty = 7,  // +stage
  bSFull = 9,   // +buffer
  bSFree = 11,  // +buffer
  bPFull = 13,
  bPVDone = 14,
  bODone = 15,
  bNum = 16
};

template <int D, bool PAGED>
__global__ void __launch_bounds__(kThreads, 1) fwd_kernel(const __grid_constant__ FwdParams p) {
  using L = FwdSmem<D>;
  constexpr int QH = D / 64;  // 64-column halves of a D-wide tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align_smem_1024(smem_raw);
  uint8_t* sQ = sm + L::kQ;
  uint8_t* sK = sm + L::kK;
  uint8_t* sV = sm + L::kV;
  uint8_t* sP = sm + L::kP;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + bNum);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const TileTask t = p.tasks[blockIdx.x];
  const int head = t.head;
  const int kvh = head / p.heads_per_kv;

  if (threadIdx.x == 0) {
    mbar_init(&bar[bQFull], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[bKFull + s], 1);
      mbar_init(&bar[bVFull + s], 1);
      mbar_init(&bar[bKEmpty + s], 1);
      mbar_init(&bar[bVEmpty + s], 1);
      mbar_init(&bar[bSFull + s], 1);
      mbar_init(&bar[bSFree + s], 4);
    }
    mbar_init(&bar[bPFull], 4);
    mbar_init(&bar[bPVDone], 1);
    mbar_init(&bar[bODone], 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS0 = tmem, tO = tmem + 256;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar[bQFull], L::kTileBytes);
      for (int h = 0; h < QH; ++h) tma_load_3d(sQ + h * 16384, &p.tm_q, &bar[bQFull], h * 64, head, t.row0);
      TileIter it;
      TileRef r;
      int i = 0;
      while (next_tile<PAGED>(p, t, it, r)) {
        const int st = i & 1;
        const uint32_t ph = (i >> 1) & 1;
        for (int kv = 0; kv < 2; ++kv) {
          uint64_t* empty = &bar[(kv == 0 ? bKEmpty : bVEmpty) + st];
          uint64_t* full = &bar[(kv == 0 ? bKFull : bVFull) + st];
          const CUtensorMap* map = kv == 0 ? &p.tm_k : &p.tm_v;
          uint8_t* dst = (kv == 0 ? sK : sV) + st * L::kTileBytes;
          if (!mbar_wait(empty, ph ^ 1, p.status, kDevTimeoutTmaEmpty)) goto producer_done;
          mbar_arrive_expect_tx(full, L::kTileBytes);
          if (!PAGED) {
            for (int h = 0; h < QH; ++h) tma_load_3d(dst + h * 16384, map, full, h * 64, kvh, r.k_row);
          } else {
            const int bs = p.block_size;
            const int ppt = BN / bs;
            for (int pg = 0; pg < ppt; ++pg) {
              int blk = (r.k_row + pg * bs) / bs;
              blk = min(blk, p.blocks_per_shard - 1);
              const int page = __ldg(&p.block_tables[(int64_t)r.shard * p.blocks_per_shard + blk]);
              for (int h = 0; h < QH; ++h)
                tma_load_4d(dst + h * 16384 + pg * bs * 128, map, full, h * 64, 0, kvh, page);
            }
          }
        }
        ++i;
      }
    producer_done:;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ UMMA issuer
    // One lane runs the loop: here that measured about 6% faster than the warp-uniform
    // loop with an elected issuing lane that the ping-pong forward and the backward use.
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(BM, BN, false, false);
      constexpr uint32_t idesc_o = idesc_bf16(BM, D, false, true);
      // base descriptors, built once; per-instruction offsets are compile-time constants
      const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dP = sdesc_sw128(smem_u32(sP), 16, 1024);
      const uint64_t dK0 = sdesc_sw128(smem_u32(sK), 16, 1024);      // stage s at + s * kTileBytes
      const uint64_t dV0 = sdesc_sw128(smem_u32(sV), 16384, 1024);
      bool ok = mbar_wait(&bar[bQFull], 0, p.status, kDevTimeoutMma);
      tc_fence_after();
      auto issue_pv = [&](int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(&bar[bPFull], j & 1, p.status, kDevTimeoutMma)) return false;
        if (!mbar_wait(&bar[bVFull + st], (j >> 1) & 1, p.status, kDevTimeoutMma)) return false;
        tc_fence_after();
        const uint64_t dv = sdesc_add(dV0, st * L::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_bf16_ss_1t(tO, sdesc_add(dP, (kk >> 2) * 16384 + (kk & 3) * 32), sdesc_add(dv, kk * 2048), idesc_o,
                       (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit_1t(&bar[bVEmpty + st]);
        umma_commit_1t(&bar[bPVDone]);
        return true;
      };
      TileIter it;
      TileRef r;
      int i = 0;
      while (ok && next_tile<PAGED>(p, t, it, r)) {
        const int st = i & 1;
        const uint32_t ph = (i >> 1) & 1;
        if (!mbar_wait(&bar[bKFull + st], ph, p.status, kDevTimeoutMma)) { ok = false; break; }
        if (!mbar_wait(&bar[bSFree + st], ph ^ 1, p.status, kDevTimeoutMma)) { ok = false; break; }
        tc_fence_after();
        const uint64_t dk = sdesc_add(dK0, st * L::kTileBytes);
        const uint32_t ts = tS0 + st * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_bf16_ss_1t(ts, sdesc_add(dQ, off), sdesc_add(dk, off), idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit_1t(&bar[bKEmpty + st]);
        umma_commit_1t(&bar[bSFull + st]);
        if (i > 0 && !issue_pv(i - 1)) { ok = false; break; }
        ++i;
      }
      if (ok && i > 0) ok = issue_pv(i - 1);
      if (i > 0) umma_commit_1t(&bar[bODone]);
      else mbar_arrive(&bar[bODone]);
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue (warps 2..5)
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int32_t qpos = t.pos0 + row;
    const float sl2 = p.scale_log2;
    const int32_t W = p.window;
    // l: exact fp32 row sum (for lse); lr: sum of the bf16-rounded P the PV product uses,
    // which normalises out so the weights applied to V sum to one exactly
    float m = -INFINITY, l = 0.f, lr = 0.f;
    bool ok = true;
    TileIter it;
    TileRef r;
    int i = 0;
    const uint32_t prow = smem_u32(sP);
    while (next_tile<PAGED>(p, t, it, r)) {
      const int sb = i & 1;
      if (!mbar_wait_warp(&bar[bSFull + sb], (i >> 1) & 1, p.status, kDevTimeoutSoftmax)) { ok = false; break; }
      tc_fence_after();
      uint32_t s[BN];
#pragma unroll
      for (int c = 0; c < BN; c += 32) tmem_ld32(tS0 + sb * 128 + lane_base + c, s + c);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[bSFree + sb]);

      if (r.need_mask && (!PAGED || p.kv_mode == kKvContiguous)) {
        // positions are linear in the column: the visible columns of this row are [lo, hi]
        int32_t hi = r.nvalid - 1, lo = 0;
        if (r.causal || W > 0) hi = min(hi, qpos - r.kpos0);
        if (W > 0) lo = max(lo, qpos - W + 1 - r.kpos0);
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c < lo || c > hi) s[c] = __float_as_uint(-INFINITY);
      } else if (r.need_mask) {
        // round-robin pages: position = page base + offset inside the page
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          const int32_t kpos = r.kpos0 + (c / p.block_size) * p.shards * p.block_size + (c % p.block_size);
          bool vis = c < r.nvalid;
          if (r.causal || W > 0) vis = vis && (kpos <= qpos);
          if (W > 0) vis = vis && (qpos - kpos < W);
          if (!vis) s[c] = __float_as_uint(-INFINITY);
        }
      }
      // row maximum of the raw scores (the scale is positive, so it commutes)
      float mraw = -INFINITY;
#pragma unroll
      for (int c = 0; c < BN; c += 2) mraw = max3f(mraw, __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
      const float mx = mraw * sl2;  // log2 units
      // running max: keep a stale max while the new one is within 2^8 (values stay bounded)
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
#pragma unroll
      for (int c = 0; c < BN; c += 2) {
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
      // PV of the previous tile must be done before O is rescaled and P is overwritten
      if (i > 0 && !mbar_wait_warp(&bar[bPVDone], (i - 1) & 1, p.status, kDevTimeoutSoftmax)) { ok = false; break; }
      tc_fence_after();
      if (__any_sync(0xffffffffu, rescale_o)) {
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          tmem_ld32(tO + lane_base + c, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + lane_base + c, o);
        }
        tmem_st_wait();
      }
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint32_t* q4 = pk + h * 32 + ch * 4;
          st_shared_v4(prow + h * 16384 + sw128_offset(row, ch), q4[0], q4[1], q4[2], q4[3]);
        }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[bPFull]);
      ++i;
    }
    // ---------------------------------------------------------------- epilogue
    if (ok && mbar_wait_warp(&bar[bODone], 0, p.status, kDevTimeoutEpilogue)) {
      tc_fence_after();
      const bool has = (l > 0.f) && (m != -INFINITY);
      const float inv_l = (has && lr > 0.f) ? 1.f / lr : 0.f;
      const float lse_b = has ? (m + __log2f(l)) * kLn2 : -INFINITY;
      const bool valid = row < t.rows;
      const int64_t orow = (int64_t)(t.row0 + row);
      const int64_t shard_off = t.aux >= 0 ? (int64_t)t.aux : 0;
      float* lse_ptr = p.lse + shard_off * p.lse_shard_stride + (int64_t)head * p.lse_stride_h + orow * p.lse_stride_t;
      const int64_t out_off = shard_off * p.out_shard_stride;
      float wa = 0.f, wb = 1.f, lse_new = lse_b;
      if (p.out_mode == kOutMerge && valid) {
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
        tmem_ld32(tO + lane_base + c, o);
        tmem_ld_wait();
        if (!valid) continue;
        if (!has) {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0u;
        }
        if (p.out_mode == kOutBf16) {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + out_off + orow * p.out_stride_t +
                               (int64_t)head * p.out_stride_h + c;
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
          float* dst = reinterpret_cast<float*>(p.out) + out_off + orow * p.out_stride_t + (int64_t)head * p.out_stride_h + c;
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            float4 v;
            v.x = __uint_as_float(o[e + 0]) * inv_l;
            v.y = __uint_as_float(o[e + 1]) * inv_l;
            v.z = __uint_as_float(o[e + 2]) * inv_l;
            v.w = __uint_as_float(o[e + 3]) * inv_l;
            if (p.out_mode == kOutMerge) {
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
int launch_fwd_t(const FwdParams& p, int grid, cudaStream_t stream) {
  auto kern = fwd_kernel<D, PAGED>;
  const uint32_t smem = FwdSmem<D>::kDynamic;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return (int)e;
  kern<<<grid, kThreads, smem, stream>>>(p);
  return (int)cudaGetLastError();
}

}  // namespace

int launch_fwd(const FwdParams& p, int head_dim, bool paged, int grid, cudaStream_t stream) {
  if (grid <= 0) return 0;
  if (head_dim == 128) return paged ? launch_fwd_t<128, true>(p, grid, stream) : launch_fwd_t<128, false>(p, grid, stream);
  if (head_dim == 64) return paged ? launch_fwd_t<64, true>(p, grid, stream) : launch_fwd_t<64, false>(p, grid, stream);
  return (int)cudaErrorInvalidValue;
}

}  // namespace cbv
