// EAGLE-3 cached attention: the per-position cache diagonals of the NeMo AutoModel ring
// page (_CachedRingAttention / _CachedZigZagRingAttention), merged into or differentiated
// against the sequence block that the ring kernels handle.
//
// The cache holds num_blocks blocks [T, Hkv, D], each at its own address; block 0 is the
// sequence (the ring's k/v),
// and every block i >= 1 contributes one key per query position t: score
// s_i = scale <q_t, k_i[t]>, value v_i[t].  All blocks form one softmax per (t, head).
//
// diag_merge_kernel: given block 0's normalised out (fp32) and lse, adds the diagonals
// with the log-sum-exp identity in one pass:
//   lse' = log(e^lse0 + sum_i e^{s_i}),   out' = out0 e^{lse0 - lse'} + sum_i v_i[t] e^{s_i - lse'}.
// diag_grad_kernel: with the merged out / lse, the closed-form gradients of the diagonal
// keys (p_i = e^{s_i - lse}, Delta = <dO, out>, dS_i = p_i (<dO, v_i[t]> - Delta)):
//   dv_i[t] += p_i dO,   dk_i[t] += scale dS_i q_t,   dq_t += scale dS_i k_i[t],
// the last added to block 0's dq (fp32) before the bf16 conversion.
//
// Both are memory-bound row kernels.  A row is served by D/8 lanes with 16-byte accesses (8 bf16
// each), so a warp holds 2 (D = 128) or 4 (D = 64) rows; dot products reduce within those lanes.
// The block count NB is a template argument so that the loops over it unroll.
#include <cuda_bf16.h>

#include "kernels.h"

namespace cbv {

namespace {

constexpr int kThreads = 256;

// sum over the L lanes of this lane's row (L a power of two, rows aligned to L lanes)
template <int L>
__device__ __forceinline__ float row_sum(float x) {
#pragma unroll
  for (int o = L / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* x) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w[j]);
    x[2 * j] = __low2float(b);
    x[2 * j + 1] = __high2float(b);
  }
}

__device__ __forceinline__ void store8(__nv_bfloat16* p, const float* x) {
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(x[2 * j], x[2 * j + 1]);
    w[j] = *reinterpret_cast<const uint32_t*>(&b);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ void load8f(const float* p, float* x) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  x[0] = a.x, x[1] = a.y, x[2] = a.z, x[3] = a.w, x[4] = b.x, x[5] = b.y, x[6] = b.z, x[7] = b.w;
}

// One row per (t, q head h).  o32 holds block 0's normalised output; out and lse get the merge.
__device__ __forceinline__ const __nv_bfloat16* blk(const void* p) { return static_cast<const __nv_bfloat16*>(p); }
__device__ __forceinline__ __nv_bfloat16* blk_w(void* p) { return static_cast<__nv_bfloat16*>(p); }

template <int D, int NB>
__global__ void __launch_bounds__(kThreads) diag_merge_kernel(const __nv_bfloat16* __restrict__ q, const CacheBlocks cb,
                                                              int64_t T, int H, int Hkv, float scale,
                                                              const float* __restrict__ o32, float* __restrict__ lse,
                                                              __nv_bfloat16* __restrict__ out) {
  constexpr int L = D / 8;  // lanes per row
  const int64_t row = ((int64_t)blockIdx.x * kThreads + threadIdx.x) / L;
  const int c = (threadIdx.x % L) * 8;  // this lane's first column
  const bool valid = row < T * H;
  const int64_t r = valid ? row : 0;  // out-of-range lanes compute on row 0 (for the shuffles) and store nothing
  const int64_t t = r / H;
  const int h = (int)(r % H);
  const int64_t kvoff = (t * Hkv + h / (H / Hkv)) * D + c;  // this row's k / v within a block
  float qv[8];
  load8(q + r * D + c, qv);
  const float l0 = lse[(int64_t)h * T + t];
  float s[NB];
  float m = l0;
#pragma unroll
  for (int i = 1; i < NB; ++i) {
    float k[8];
    load8(blk(cb.k[i]) + kvoff, k);
    float d = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) d = fmaf(qv[e], k[e], d);
    s[i] = scale * row_sum<L>(d);
    m = fmaxf(m, s[i]);
  }
  float z = l0 == -INFINITY ? 0.f : __expf(l0 - m);
#pragma unroll
  for (int i = 1; i < NB; ++i) z += __expf(s[i] - m);
  const float ln = m + __logf(z);
  const float w0 = l0 == -INFINITY ? 0.f : __expf(l0 - ln);
  float acc[8];
  load8f(o32 + r * D + c, acc);
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] *= w0;
#pragma unroll
  for (int i = 1; i < NB; ++i) {
    float v[8];
    load8(blk(cb.v[i]) + kvoff, v);
    const float w = __expf(s[i] - ln);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, v[e], acc[e]);
  }
  if (!valid) return;
  store8(out + r * D + c, acc);
  if (c == 0) lse[(int64_t)h * T + t] = ln;
}

// One row per (t, kv head).  Pass 1 walks the kv head's G q heads: dq (block 0's fp32 part plus
// the diagonal terms) is written, and every (q head, block) pair leaves p and dS in shared memory.
// Pass 2 forms each block's dk / dv from them, re-reading q and dO (now in L1).
template <int D, int NB>
__global__ void __launch_bounds__(kThreads) diag_grad_kernel(
    const __nv_bfloat16* __restrict__ q, const CacheBlocks cb, int64_t T, int H, int Hkv, float scale,
    const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ out, const float* __restrict__ lse,
    const float* __restrict__ dq_acc, const unsigned long long* __restrict__ dq_fixed, __nv_bfloat16* __restrict__ dq) {
  constexpr int L = D / 8;
  constexpr int kRows = kThreads / L;  // rows per CTA
  extern __shared__ float2 pds[];      // [kRows][G][NB - 1] of {p, dS}
  const int G = H / Hkv;
  const int lr = threadIdx.x / L;      // row within the CTA
  const int64_t row = (int64_t)blockIdx.x * kRows + lr;
  const int c = (threadIdx.x % L) * 8;
  const bool valid = row < T * Hkv;
  const int64_t r = valid ? row : 0;
  const int64_t t = r / Hkv;
  const int kh = (int)(r % Hkv);
  const int64_t kvoff = r * D + c;
  float2* my = pds + (size_t)lr * G * (NB - 1);
  for (int g = 0; g < G; ++g) {
    const int h = kh * G + g;
    const int64_t qoff = (t * H + h) * D + c;
    float qv[8], dov[8], ov[8], acc[8];
    load8(q + qoff, qv);
    load8(dout + qoff, dov);
    load8(out + qoff, ov);
    if (dq_fixed) {  // deterministic mode: 64-bit fixed point in units of 2^-32, quarter-major layout
      const unsigned long long* f = dq_fixed + fixed_index(t, h, c, fixed_tpad(T), D);
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const ulonglong2 u = __ldg(reinterpret_cast<const ulonglong2*>(f + e));
        acc[e] = __ll2float_rn((long long)u.x) * 2.3283064365386963e-10f;
        acc[e + 1] = __ll2float_rn((long long)u.y) * 2.3283064365386963e-10f;
      }
    } else {
      load8f(dq_acc + qoff, acc);
    }
    float delta = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) delta = fmaf(dov[e], ov[e], delta);
    delta = row_sum<L>(delta);
    const float l = lse[(int64_t)h * T + t];
#pragma unroll
    for (int i = 1; i < NB; ++i) {
      float k[8], v[8];
      load8(blk(cb.k[i]) + kvoff, k);
      load8(blk(cb.v[i]) + kvoff, v);
      float sd = 0.f, pd = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        sd = fmaf(qv[e], k[e], sd);
        pd = fmaf(dov[e], v[e], pd);
      }
      sd = row_sum<L>(sd);
      pd = row_sum<L>(pd);
      const float p = l == -INFINITY ? 0.f : __expf(scale * sd - l);
      const float ds = p * (pd - delta);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = fmaf(scale * ds, k[e], acc[e]);
      if (c == 0) my[g * (NB - 1) + i - 1] = make_float2(p, ds);
    }
    if (valid) store8(dq + qoff, acc);
  }
  __syncwarp();
  if (!valid) return;
#pragma unroll
  for (int i = 1; i < NB; ++i) {
    float dk[8] = {}, dv[8] = {};
    for (int g = 0; g < G; ++g) {
      const int64_t qoff = (t * H + kh * G + g) * D + c;
      const float2 pd = my[g * (NB - 1) + i - 1];
      float qv[8], dov[8];
      load8(q + qoff, qv);
      load8(dout + qoff, dov);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        dk[e] = fmaf(scale * pd.y, qv[e], dk[e]);
        dv[e] = fmaf(pd.x, dov[e], dv[e]);
      }
    }
    store8(blk_w(cb.dk[i]) + kvoff, dk);
    store8(blk_w(cb.dv[i]) + kvoff, dv);
  }
}

template <int D, int NB>
int merge_nb(const void* q, const CacheBlocks& cb, int64_t T, int H, int Hkv, float scale, const float* o32,
             float* lse, void* out, cudaStream_t stream) {
  const int64_t lanes = T * H * (D / 8);
  const int64_t blocks = (lanes + kThreads - 1) / kThreads;
  diag_merge_kernel<D, NB><<<blocks, kThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(q), cb, T, H, Hkv,
                                                             scale, o32, lse, static_cast<__nv_bfloat16*>(out));
  return launched();
}

template <int D, int NB>
int grad_nb(const void* q, const CacheBlocks& cb, int64_t T, int H, int Hkv, float scale, const void* dout,
            const void* out, const float* lse, const float* dq_acc, const unsigned long long* dq_fixed, void* dq,
            cudaStream_t stream) {
  constexpr int kRows = kThreads / (D / 8);
  const size_t smem = (size_t)kRows * (H / Hkv) * (NB - 1) * sizeof(float2);
  auto kern = diag_grad_kernel<D, NB>;
  if (smem > 48 * 1024) {
    if (smem > 227 * 1024) return (int)cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return (int)e;
  }
  const int64_t blocks = (T * Hkv + kRows - 1) / kRows;
  auto c = [](const void* p) { return static_cast<const __nv_bfloat16*>(p); };
  kern<<<blocks, kThreads, smem, stream>>>(c(q), cb, T, H, Hkv, scale, c(dout), c(out), lse, dq_acc, dq_fixed,
                                           static_cast<__nv_bfloat16*>(dq));
  return launched();
}

template <int D>
int merge_d(int nb, const void* q, const CacheBlocks& cb, int64_t T, int H, int Hkv, float scale, const float* o32,
            float* lse, void* out, cudaStream_t s) {
  switch (nb) {
    case 2: return merge_nb<D, 2>(q, cb, T, H, Hkv, scale, o32, lse, out, s);
    case 3: return merge_nb<D, 3>(q, cb, T, H, Hkv, scale, o32, lse, out, s);
    case 4: return merge_nb<D, 4>(q, cb, T, H, Hkv, scale, o32, lse, out, s);
    case 5: return merge_nb<D, 5>(q, cb, T, H, Hkv, scale, o32, lse, out, s);
    case 6: return merge_nb<D, 6>(q, cb, T, H, Hkv, scale, o32, lse, out, s);
    case 7: return merge_nb<D, 7>(q, cb, T, H, Hkv, scale, o32, lse, out, s);
    case 8: return merge_nb<D, 8>(q, cb, T, H, Hkv, scale, o32, lse, out, s);
    default: return (int)cudaErrorInvalidValue;
  }
}

template <int D>
int grad_d(int nb, const void* q, const CacheBlocks& cb, int64_t T, int H, int Hkv, float scale, const void* dout,
           const void* out, const float* lse, const float* dq_acc, const unsigned long long* dq_fixed, void* dq,
           cudaStream_t s) {
  switch (nb) {
    case 2: return grad_nb<D, 2>(q, cb, T, H, Hkv, scale, dout, out, lse, dq_acc, dq_fixed, dq, s);
    case 3: return grad_nb<D, 3>(q, cb, T, H, Hkv, scale, dout, out, lse, dq_acc, dq_fixed, dq, s);
    case 4: return grad_nb<D, 4>(q, cb, T, H, Hkv, scale, dout, out, lse, dq_acc, dq_fixed, dq, s);
    case 5: return grad_nb<D, 5>(q, cb, T, H, Hkv, scale, dout, out, lse, dq_acc, dq_fixed, dq, s);
    case 6: return grad_nb<D, 6>(q, cb, T, H, Hkv, scale, dout, out, lse, dq_acc, dq_fixed, dq, s);
    case 7: return grad_nb<D, 7>(q, cb, T, H, Hkv, scale, dout, out, lse, dq_acc, dq_fixed, dq, s);
    case 8: return grad_nb<D, 8>(q, cb, T, H, Hkv, scale, dout, out, lse, dq_acc, dq_fixed, dq, s);
    default: return (int)cudaErrorInvalidValue;
  }
}

}  // namespace

int launch_diag_merge(const void* q, const CacheBlocks& cb, int nb, int64_t T, int H, int Hkv, int D, float scale,
                      const float* o32, float* lse, void* out, cudaStream_t stream) {
  if (T * H == 0) return 0;
  if (D == 128) return merge_d<128>(nb, q, cb, T, H, Hkv, scale, o32, lse, out, stream);
  if (D == 64) return merge_d<64>(nb, q, cb, T, H, Hkv, scale, o32, lse, out, stream);
  return (int)cudaErrorInvalidValue;
}

int launch_diag_grad(const void* q, const CacheBlocks& cb, int nb, int64_t T, int H, int Hkv, int D, float scale,
                     const void* dout, const void* out, const float* lse, const float* dq_acc,
                     const unsigned long long* dq_fixed, void* dq, cudaStream_t stream) {
  if (T * Hkv == 0) return 0;
  if (D == 128) return grad_d<128>(nb, q, cb, T, H, Hkv, scale, dout, out, lse, dq_acc, dq_fixed, dq, stream);
  if (D == 64) return grad_d<64>(nb, q, cb, T, H, Hkv, scale, dout, out, lse, dq_acc, dq_fixed, dq, stream);
  return (int)cudaErrorInvalidValue;
}

}  // namespace cbv
