// One-query-per-sequence GQA varlen decode (qsa_fa_fallback.py, SM121 recipe:
// _varlen_one_q_attn_kernel / triton_varlen_attn_func).
//
// Sequence s has one query row cu_q[s] and keys [cu_k[s], cu_k[s+1]); q head h
// reads kv head h / (HQ/HKV); no mask; an empty key range gives zeros.  The
// offsets are read on the device, so the launch needs nothing from the host per
// call and stays valid when cu_seqlens change between graph replays.
//
// The pass is HBM-bound: every K/V byte is read once.  One CTA serves one
// sequence and up to four kv heads; TMA streams 32-key tiles of K and V for the
// four heads into a 3-stage shared-memory ring (128B swizzle); warp w computes kv
// head w%4 over key half w/4 of every tile.  The G = HQ/HKV query heads sharing a
// kv head form the 16 rows of an m16n8k16 tensor-core tile (G <= 16), so the
// score and value contractions run on the tensor pipe and the CUDA cores only do
// the online softmax.  The two key halves are merged with the log-sum-exp
// identity at the end.
#include "kernels.h"
#include "ptx.cuh"

namespace cbv {

namespace {

constexpr int kDecKeys = 32;     // keys per tile
constexpr int kDecHeads = 4;     // kv heads per CTA
constexpr int kDecStages = 3;
constexpr int kDecThreads = 256;

__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

template <int D>
struct DecSmem {
  static constexpr uint32_t kHead = kDecKeys * 128;               // 32 rows x 64 columns of one head
  static constexpr uint32_t kHalfMax = kDecHeads * kHead;          // one 64-column half, up to 4 heads
  static constexpr uint32_t kTileMax = (D / 64) * kHalfMax;        // K (or V) of one tile
  static constexpr uint32_t kStage = 2 * kTileMax;
  static constexpr uint32_t kBars = kDecStages * kStage;
  static constexpr uint32_t kEnd = kBars + 128;
  static constexpr uint32_t kDynamic = kEnd + 1024;
};

template <int D>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(const __grid_constant__ DecodeParams p) {
  using L = DecSmem<D>;
  constexpr int KS = D / 16;  // k16 steps over the head dim
  constexpr int ND = D / 8;   // n8 blocks over the head dim
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align_smem_1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L::kBars);
  uint64_t* empty = full + kDecStages;

  const int seq = blockIdx.x;
  const int group = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hsub = warp & 3;   // kv head within the group
  const int khalf = warp >> 2; // which 16 keys of each tile
  const int hpc = p.heads_per_cta;  // kv heads per CTA (4, 2 or 1: divides HKV)
  const int kvh = group * hpc + hsub;
  const int G = p.hq / p.hkv;
  const bool active = hsub < hpc;
  const uint32_t half_bytes = hpc * L::kHead;
  const uint32_t tile_bytes = (D / 64) * half_bytes;

  int qrow = __ldg(&p.cu_q[seq]);
  int k_start = __ldg(&p.cu_k[seq]);
  int k_end = __ldg(&p.cu_k[seq + 1]);
  // the offsets are read here, not checked on the host (they may change between graph replays): a
  // sequence whose offsets leave the tensors is reported and skipped
  const bool bad = qrow < 0 || qrow >= p.total_q || k_start < 0 || k_end > p.total_k || k_end < k_start;
  if (bad) {
    if (threadIdx.x == 0) atomicCAS(p.status, 0, kDevBadOffsets);
    return;
  }
  const int nkeys = max(0, k_end - k_start);
  const int ntiles = (nkeys + kDecKeys - 1) / kDecKeys;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecThreads / 32);
    }
    fence_mbar_init();
  }
  __syncthreads();

  auto issue = [&](int tile) {
    const int st = tile % kDecStages;
    uint8_t* base = sm + st * L::kStage;
    mbar_arrive_expect_tx(&full[st], 2 * tile_bytes);
    const int row = k_start + tile * kDecKeys;
    for (int h = 0; h < D / 64; ++h) {
      tma_load_3d(base + h * half_bytes, &p.tm_k, &full[st], h * 64, row, group * hpc);
      tma_load_3d(base + tile_bytes + h * half_bytes, &p.tm_v, &full[st], h * 64, row, group * hpc);
    }
  };
  if (threadIdx.x == 0) {
    for (int tl = 0; tl < min(ntiles, kDecStages); ++tl) issue(tl);
  }

  // Q fragments (A operand, rows = the G query heads of this kv head, zero-padded to 16)
  const int g = lane >> 2, tq = lane & 3;
  uint32_t qa[KS][4];
  {
    const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(p.q) + (int64_t)qrow * p.hq * D;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = g + ((e & 1) ? 8 : 0);
        const int c = ks * 16 + tq * 2 + ((e & 2) ? 8 : 0);
        uint32_t v = 0;
        if (active && r < G) v = __ldg(reinterpret_cast<const uint32_t*>(qb + (int64_t)(kvh * G + r) * D + c));
        qa[ks][e] = v;
      }
    }
  }

  float o[ND][4];
#pragma unroll
  for (int n = 0; n < ND; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // rows g and g+8
  const float sl2 = p.scale_log2;
  bool ok = true;

  for (int tl = 0; tl < ntiles; ++tl) {
    const int st = tl % kDecStages;
    if (!mbar_wait_warp(&full[st], (tl / kDecStages) & 1, p.status, kDevTimeoutTmaFull)) { ok = false; break; }
    const uint32_t kbase = smem_u32(sm + st * L::kStage) + (active ? hsub : 0) * L::kHead;
    const uint32_t vbase = kbase + tile_bytes;
    // scores: 16 rows x 16 keys (this warp's key half), two n8 blocks
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) {
      const int krow = khalf * 16 + nb * 8 + (lane & 7);
#pragma unroll
      for (int kp = 0; kp < KS; kp += 2) {
        const int chunk = kp * 2 + (lane >> 3);  // 16-byte chunk along D (0..D/8-1)
        const uint32_t addr = kbase + (chunk >> 3) * half_bytes + sw128_offset(krow, chunk & 7);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(addr, b0, b1, b2, b3);
        mma_bf16_16816(s[nb], qa[kp], b0, b1);
        mma_bf16_16816(s[nb], qa[kp + 1], b2, b3);
      }
    }
    // mask keys past the sequence end, scale to log2 units
    const int kbase_idx = tl * kDecKeys + khalf * 16;
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = kbase_idx + nb * 8 + tq * 2 + (e & 1);
        const float v = key < nkeys ? s[nb][e] * sl2 : -INFINITY;
        s[nb][e] = v;
        if (e < 2) mx0 = fmaxf(mx0, v);
        else mx1 = fmaxf(mx1, v);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float a0 = (m0 == -INFINITY) ? 0.f : ex2_approx(m0 - mn0);
    const float a1 = (m1 == -INFINITY) ? 0.f : ex2_approx(m1 - mn1);
    const float sub0 = (mn0 == -INFINITY) ? 0.f : mn0, sub1 = (mn1 == -INFINITY) ? 0.f : mn1;
    float rs0 = 0.f, rs1 = 0.f;
    uint32_t pa[4];
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) {
      const float p0 = ex2_approx(s[nb][0] - sub0), p1 = ex2_approx(s[nb][1] - sub0);
      const float p2 = ex2_approx(s[nb][2] - sub1), p3 = ex2_approx(s[nb][3] - sub1);
      rs0 += p0 + p1;
      rs1 += p2 + p3;
      pa[nb * 2 + 0] = pack_bf16x2(p0, p1);
      pa[nb * 2 + 1] = pack_bf16x2(p2, p3);
    }
    l0 = l0 * a0 + rs0;
    l1 = l1 * a1 + rs1;
    m0 = mn0;
    m1 = mn1;
#pragma unroll
    for (int n = 0; n < ND; ++n) {
      o[n][0] *= a0;
      o[n][1] *= a0;
      o[n][2] *= a1;
      o[n][3] *= a1;
    }
    // O += P V over this warp's 16 keys
    {
      const int vrow = khalf * 16 + (lane & 7) + ((lane & 8) ? 8 : 0);
#pragma unroll
      for (int nd = 0; nd < ND; nd += 2) {
        const int chunk = nd + (lane >> 4);
        const uint32_t addr = vbase + (chunk >> 3) * half_bytes + sw128_offset(vrow, chunk & 7);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(addr, b0, b1, b2, b3);
        mma_bf16_16816(o[nd], pa, b0, b1);
        mma_bf16_16816(o[nd + 1], pa, b2, b3);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
    if (threadIdx.x == 0 && tl + kDecStages < ntiles) {
      if (!mbar_wait(&empty[st], (tl / kDecStages) & 1, p.status, kDevTimeoutTmaEmpty)) { ok = false; }
      else issue(tl + kDecStages);
    }
  }
  // full row sums across the quad
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

  // merge the two key halves through shared memory (the stage ring is free now)
  __syncthreads();
  float* red = reinterpret_cast<float*>(sm);  // [4 heads][16 rows][D] + m, l
  float* red_ml = red + kDecHeads * 16 * D;
  if (khalf == 1) {
#pragma unroll
    for (int n = 0; n < ND; ++n) {
      const int c = n * 8 + tq * 2;
      red[(hsub * 16 + g) * D + c] = o[n][0];
      red[(hsub * 16 + g) * D + c + 1] = o[n][1];
      red[(hsub * 16 + g + 8) * D + c] = o[n][2];
      red[(hsub * 16 + g + 8) * D + c + 1] = o[n][3];
    }
    if (tq == 0) {
      red_ml[(hsub * 16 + g) * 2 + 0] = m0;
      red_ml[(hsub * 16 + g) * 2 + 1] = l0;
      red_ml[(hsub * 16 + g + 8) * 2 + 0] = m1;
      red_ml[(hsub * 16 + g + 8) * 2 + 1] = l1;
    }
  }
  __syncthreads();
  if (khalf == 0 && active && ok) {
    const float mb0 = red_ml[(hsub * 16 + g) * 2 + 0], lb0 = red_ml[(hsub * 16 + g) * 2 + 1];
    const float mb1 = red_ml[(hsub * 16 + g + 8) * 2 + 0], lb1 = red_ml[(hsub * 16 + g + 8) * 2 + 1];
    const float M0 = fmaxf(m0, mb0), M1 = fmaxf(m1, mb1);
    const float wa0 = (m0 == -INFINITY) ? 0.f : ex2_approx(m0 - M0), wb0 = (mb0 == -INFINITY) ? 0.f : ex2_approx(mb0 - M0);
    const float wa1 = (m1 == -INFINITY) ? 0.f : ex2_approx(m1 - M1), wb1 = (mb1 == -INFINITY) ? 0.f : ex2_approx(mb1 - M1);
    const float L0 = l0 * wa0 + lb0 * wb0, L1 = l1 * wa1 + lb1 * wb1;
    const float i0 = L0 > 0.f ? 1.f / L0 : 0.f, i1 = L1 > 0.f ? 1.f / L1 : 0.f;
    __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(p.out) + (int64_t)qrow * p.hq * D;
#pragma unroll
    for (int n = 0; n < ND; ++n) {
      const int c = n * 8 + tq * 2;
      if (g < G) {
        const float x0 = (o[n][0] * wa0 + red[(hsub * 16 + g) * D + c] * wb0) * i0;
        const float x1 = (o[n][1] * wa0 + red[(hsub * 16 + g) * D + c + 1] * wb0) * i0;
        *reinterpret_cast<uint32_t*>(ob + (int64_t)(kvh * G + g) * D + c) = pack_bf16x2(x0, x1);
      }
      if (g + 8 < G) {
        const float x2 = (o[n][2] * wa1 + red[(hsub * 16 + g + 8) * D + c] * wb1) * i1;
        const float x3 = (o[n][3] * wa1 + red[(hsub * 16 + g + 8) * D + c + 1] * wb1) * i1;
        *reinterpret_cast<uint32_t*>(ob + (int64_t)(kvh * G + g + 8) * D + c) = pack_bf16x2(x2, x3);
      }
    }
  }
}

template <int D>
int launch_decode_t(const DecodeParams& p, cudaStream_t stream) {
  auto kern = decode_kernel<D>;
  const uint32_t smem = DecSmem<D>::kDynamic;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return (int)e;
  dim3 grid(p.num_seqs, p.hkv / p.heads_per_cta);
  if (const int ev = kernel_event_start(stream)) return ev;
  kern<<<grid, kDecThreads, smem, stream>>>(p);
  const int rc = launched();
  if (rc) return rc;
  return kernel_event_stop(stream);
}

}  // namespace

int launch_decode(const DecodeParams& p, cudaStream_t stream) {
  if (p.num_seqs <= 0) return 0;
  if (p.head_dim == 128) return launch_decode_t<128>(p, stream);
  if (p.head_dim == 64) return launch_decode_t<64>(p, stream);
  return (int)cudaErrorInvalidValue;
}

}  // namespace cbv
