// Memory-bound helper kernels: the standalone online-softmax merge, the backward
// preprocess (Delta = rowsum(dO * O)) and the fp32 -> bf16 conversion.
#include <cstring>

#include "kernels.h"
#include "ptx.cuh"

namespace cbv {

namespace {

// One warp per (token, head) row; every lane owns D/32 consecutive elements.
//
// NeMo AutoModel, zigzag_ring_attention, update_out_and_lse (and ring_attention,
// _update_out_and_lse): with w = sigmoid(block_lse - lse),
//   out' = out - w (out - block_out),  lse' = lse - logsigmoid(lse - block_lse),
// evaluated here as lse' = m + log(e^(lse-m) + e^(blse-m)), m = max(lse, blse), and
// out' = out e^(lse-lse') + block_out e^(blse-lse'), which is the same quantity;
// a side at -inf is the identity of the merge.
template <int D, bool BF16_IN>
__global__ void __launch_bounds__(256) merge_kernel(float* __restrict__ out, float* __restrict__ lse,
                                                    const void* __restrict__ block_out,
                                                    const float* __restrict__ block_lse, float* __restrict__ weight,
                                                    int64_t seqlen, int heads) {
  // D/8 lanes per (token, head) row, 8 elements each; rows numbered head-major so that
  // consecutive rows read and write consecutive lse entries
  constexpr int L = D / 8;
  const int64_t rowid = ((int64_t)blockIdx.x * 256 + threadIdx.x) / L;
  const int c = (threadIdx.x % L) * 8;
  // every lane of a row reads lse[li] before one of them overwrites it: no early exit, and a
  // warp barrier between the reads and the write
  const bool valid = rowid < seqlen * heads;
  const int64_t r = valid ? rowid : 0;
  const int64_t h = r / seqlen, tok = r % seqlen;
  const int64_t li = r;  // == h * seqlen + tok
  const float a = lse[li];
  const float b = block_lse[li];
  const float m = fmaxf(a, b);
  float wa, wb, nl, w;
  if (m == -INFINITY) {
    wa = 1.f;
    wb = 0.f;
    nl = -INFINITY;
    w = 0.f;
  } else {
    nl = m + __logf(__expf(a - m) + __expf(b - m));
    wa = __expf(a - nl);
    wb = __expf(b - nl);
    w = wb;  // sigmoid(b - a) with the pre-merge lse
  }
  const int64_t off = (tok * heads + h) * D + c;
  float4* o = reinterpret_cast<float4*>(out + off);
  float4 x0 = o[0], x1 = o[1];
  float y[8];
  if (BF16_IN) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(block_out) + off));
    const uint32_t wds[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&wds[j]);
      y[2 * j] = __low2float(v);
      y[2 * j + 1] = __high2float(v);
    }
  } else {
    const float4* bo = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(block_out) + off);
    const float4 v0 = __ldg(bo), v1 = __ldg(bo + 1);
    y[0] = v0.x, y[1] = v0.y, y[2] = v0.z, y[3] = v0.w, y[4] = v1.x, y[5] = v1.y, y[6] = v1.z, y[7] = v1.w;
  }
  x0 = make_float4(x0.x * wa + y[0] * wb, x0.y * wa + y[1] * wb, x0.z * wa + y[2] * wb, x0.w * wa + y[3] * wb);
  x1 = make_float4(x1.x * wa + y[4] * wb, x1.y * wa + y[5] * wb, x1.z * wa + y[6] * wb, x1.w * wa + y[7] * wb);
  if (valid) {
    o[0] = x0;
    o[1] = x1;
  }
  __syncwarp();
  if (valid && c == 0) {
    lse[li] = nl;
    if (weight) weight[li] = w;
  }
}

// Backward preprocess: Delta_i = <dO_i, O_i> with the merged (bf16) output, and the
// merged lse in log2 units, both laid out [H, t_pad] for the backward's row loads; with
// dq_zero, the row's fp32 dq accumulator is zeroed in the same pass.  D/8 lanes per
// (token, head) row with 16-byte accesses; rows are numbered head-major, so consecutive rows
// read consecutive lse entries and write consecutive row pairs.
template <int D>
__global__ void __launch_bounds__(256) delta_kernel(const __nv_bfloat16* __restrict__ dout,
                                                    const __nv_bfloat16* __restrict__ out,
                                                    const float* __restrict__ lse, float2* __restrict__ rows,
                                                    float* __restrict__ dq_zero, int64_t total, int64_t t_pad,
                                                    int heads) {
  constexpr int L = D / 8;  // lanes per row
  const int64_t rowid = ((int64_t)blockIdx.x * 256 + threadIdx.x) / L;
  const int c = (threadIdx.x % L) * 8;
  const bool valid = rowid < total * heads;
  const int64_t h = valid ? rowid / total : 0;
  const int64_t tok = valid ? rowid % total : 0;
  const int64_t off = (tok * heads + h) * D + c;
  const uint4 ua = __ldg(reinterpret_cast<const uint4*>(dout + off));
  const uint4 ub = __ldg(reinterpret_cast<const uint4*>(out + off));
  const uint32_t wa[4] = {ua.x, ua.y, ua.z, ua.w}, wb[4] = {ub.x, ub.y, ub.z, ub.w};
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(&wa[j]);
    const __nv_bfloat162 y = *reinterpret_cast<const __nv_bfloat162*>(&wb[j]);
    s = fmaf(__low2float(x), __low2float(y), s);
    s = fmaf(__high2float(x), __high2float(y), s);
  }
#pragma unroll
  for (int o = L / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (!valid) return;
  if (dq_zero) {
    float4* z = reinterpret_cast<float4*>(dq_zero + off);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (c == 0) {
    // A row that sees no key at all has lse = -inf; it is masked in every block, and storing a
    // finite value keeps exp2(-inf - lse) at 0 in the backward's masked tiles.  The pad rows
    // [total, t_pad) are zeroed: a row box may read them.
    const float l = lse[h * total + tok];
    rows[h * t_pad + tok] = make_float2(l == -INFINITY ? 0.f : l * 1.4426950408889634f, s);
    for (int64_t e = total + tok; e < t_pad; e += total) rows[h * t_pad + e] = make_float2(0.f, 0.f);
  }
}

__global__ void __launch_bounds__(256) convert_kernel(const float4* __restrict__ src, uint2* __restrict__ dst,
                                                      int64_t n4, float mul) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = src[i];
    dst[i] = make_uint2(pack_bf16x2(v.x * mul, v.y * mul), pack_bf16x2(v.z * mul, v.w * mul));
  }
}

// 64-bit fixed point in units of 2^-32: the integer rounds to the nearest fp32, and the power-of-two
// scale is exact.
__device__ __forceinline__ float fixed_to_float(unsigned long long x) {
  return __ll2float_rn((long long)x) * 2.3283064365386963e-10f;
}

// One thread per pair of adjacent head dims (never split across a quarter: D/4 is even).
__global__ void __launch_bounds__(256) fixed_to_bf16_kernel(const unsigned long long* __restrict__ src,
                                                            __nv_bfloat162* __restrict__ dst, int64_t T, int H,
                                                            int D, int64_t tpad) {
  const int64_t n2 = T * H * D / 2;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n2; i += (int64_t)gridDim.x * blockDim.x) {
    const int d = (int)(2 * i % D);
    const int64_t th = 2 * i / D;
    const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(src + fixed_index(th / H, (int)(th % H), d, tpad, D));
    dst[i] = __floats2bfloat162_rn(fixed_to_float(v.x), fixed_to_float(v.y));
  }
}

__global__ void __launch_bounds__(256) fixed_add_f32_kernel(const unsigned long long* __restrict__ src,
                                                            float2* __restrict__ dst, int64_t T, int H, int D,
                                                            int64_t tpad) {
  const int64_t n2 = T * H * D / 2;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n2; i += (int64_t)gridDim.x * blockDim.x) {
    const int d = (int)(2 * i % D);
    const int64_t th = 2 * i / D;
    const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(src + fixed_index(th / H, (int)(th % H), d, tpad, D));
    float2 o = dst[i];
    o.x += fixed_to_float(v.x);
    o.y += fixed_to_float(v.y);
    dst[i] = o;
  }
}

// [H, S, D] fp32 -> [H, D, S] bf16 through a 32 x 32 shared-memory tile: reads run along D,
// writes along S, both coalesced.  Block (32, 8); grid (ceil(S/32), D/32, H).
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const float* __restrict__ src,
                                                             __nv_bfloat16* __restrict__ dst, int64_t S, int D) {
  __shared__ float tile[32][33];
  const int64_t s0 = (int64_t)blockIdx.x * 32;
  const int d0 = blockIdx.y * 32;
  const int64_t h = blockIdx.z;
  const float* in = src + h * S * D;
  __nv_bfloat16* outp = dst + h * S * D;
  for (int r = threadIdx.y; r < 32; r += 8) {
    const int64_t s = s0 + r;
    if (s < S) tile[r][threadIdx.x] = in[s * D + d0 + threadIdx.x];
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += 8) {
    const int64_t s = s0 + threadIdx.x;
    if (s < S) outp[(int64_t)(d0 + r) * S + s] = __float2bfloat16_rn(tile[threadIdx.x][r]);
  }
}

constexpr int kInlineBytes = 30 * 1024;
struct InlineChunk {
  uint4* dst;
  uint32_t n16;  // 16-byte words
  uint32_t pad;
  uint4 data[kInlineBytes / 16];
};

__global__ void __launch_bounds__(256) inline_copy_kernel(const __grid_constant__ InlineChunk c) {
  for (uint32_t i = threadIdx.x; i < c.n16; i += blockDim.x) c.dst[i] = c.data[i];
}

// The usual case, a schedule image that fits one payload: one launch both writes the image to
// the workspace (block 0) and expands the task list, reading the groups and tiles straight from
// its own parameters; it also clears the call's status word.  The payload comes in three sizes,
// so that a small schedule does not pay for uploading 30 KB of launch parameters.
template <int kBytes>
struct ScheduleChunk {
  uint4* dst;                // the image's place in the workspace
  TileTask* tasks;           // the expanded task list
  int* status;               // cleared by the first thread (may be null)
  uint32_t n16;              // image size, 16-byte words
  uint32_t off_tiles;        // byte offset of the tiles in the image (the groups start at 0)
  int32_t ngroups, ntasks;
  uint4 data[kBytes / 16];
};

template <int kBytes>
__global__ void __launch_bounds__(256) schedule_kernel(const __grid_constant__ ScheduleChunk<kBytes> c) {
  if (blockIdx.x == 0) {
    if (threadIdx.x == 0 && c.status) *c.status = 0;
    for (uint32_t i = threadIdx.x; i < c.n16; i += blockDim.x) c.dst[i] = c.data[i];
  }
  const PlanGroup* groups = reinterpret_cast<const PlanGroup*>(c.data);
  const TileTask* tiles = reinterpret_cast<const TileTask*>(reinterpret_cast<const unsigned char*>(c.data) + c.off_tiles);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < c.ntasks; i += gridDim.x * blockDim.x) {
    int lo = 0, hi = c.ngroups - 1;  // the last group whose first task is <= i
    while (lo < hi) {
      const int mid = (lo + hi + 1) / 2;
      if (groups[mid].first_task <= i) lo = mid;
      else hi = mid - 1;
    }
    const PlanGroup g = groups[lo];
    const int local = i - g.first_task;
    TileTask t = tiles[g.first_tile + local % g.ntiles];
    t.head = local / g.ntiles;
    c.tasks[i] = t;
  }
}

template <int kBytes>
int launch_schedule_t(void* image_dst, const void* image, size_t bytes, size_t off_tiles, int ngroups, TileTask* tasks,
                      int ntasks, int* status, cudaStream_t stream) {
  ScheduleChunk<kBytes> c;
  c.dst = static_cast<uint4*>(image_dst);
  c.tasks = tasks;
  c.status = status;
  c.n16 = (uint32_t)(bytes / 16);
  c.off_tiles = (uint32_t)off_tiles;
  c.ngroups = ngroups;
  c.ntasks = ntasks;
  memcpy(c.data, image, bytes);
  const int blocks = std::min((ntasks + 255) / 256, 148 * 4);
  schedule_kernel<kBytes><<<blocks, 256, 0, stream>>>(c);
  return launched();
}

__global__ void __launch_bounds__(256) expand_tasks_kernel(const PlanGroup* __restrict__ groups, int ngroups,
                                                           const TileTask* __restrict__ tiles,
                                                           TileTask* __restrict__ tasks, int ntasks) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < ntasks; i += gridDim.x * blockDim.x) {
    int lo = 0, hi = ngroups - 1;  // the last group whose first task is <= i
    while (lo < hi) {
      const int mid = (lo + hi + 1) / 2;
      if (groups[mid].first_task <= i) lo = mid;
      else hi = mid - 1;
    }
    const PlanGroup g = groups[lo];
    const int local = i - g.first_task;
    TileTask t = tiles[g.first_tile + local % g.ntiles];
    t.head = local / g.ntiles;
    tasks[i] = t;
  }
}

// The two halves of a split prefill task attend disjoint parts of the keys for the same q rows.
// Their normalised partials combine by the log-sum-exp identity (update_out_and_lse):
// lse = log(e^lse0 + e^lse1) and out = e^(lse0 - lse) out0 + e^(lse1 - lse) out1, rounded
// to the bf16 output (head-major rows; a head-dim stride > 1 gives the transposed layout).
// A half at -inf has weight 0; both at -inf give out = 0 and lse = -inf.
template <int D>
__global__ void __launch_bounds__(256) merge_halves_kernel(const TileTask* __restrict__ tasks,
                                                           const float* __restrict__ part,
                                                           const float* __restrict__ part_lse, int64_t part_stride,
                                                           int64_t lse_part_stride, int64_t q_len,
                                                           __nv_bfloat16* __restrict__ out, int64_t out_stride_h,
                                                           int64_t out_stride_t, int64_t out_stride_d,
                                                           float* __restrict__ lse) {
  constexpr int L = D / 8;         // lanes per row, 8 elements each
  constexpr int kRows = 256 / L;   // rows per block
  const TileTask t = tasks[blockIdx.x];
  const int r = blockIdx.y * kRows + (int)threadIdx.x / L;
  if (r >= t.rows) return;
  const int c = ((int)threadIdx.x % L) * 8;
  const int64_t row = (int64_t)t.row0 + r;
  const int64_t li = (int64_t)t.head * q_len + row;
  const float l0 = part_lse[li], l1 = part_lse[lse_part_stride + li];
  const float m = fmaxf(l0, l1);
  float w0 = 0.f, w1 = 0.f, nl = -INFINITY;
  if (m != -INFINITY) {
    nl = m + __logf(__expf(l0 - m) + __expf(l1 - m));
    w0 = __expf(l0 - nl);
    w1 = __expf(l1 - nl);
  }
  const float4* a = reinterpret_cast<const float4*>(part + li * D + c);
  const float4* b = reinterpret_cast<const float4*>(part + part_stride + li * D + c);
  const float4 a0 = __ldg(a), a1 = __ldg(a + 1), b0 = __ldg(b), b1 = __ldg(b + 1);
  const float v[8] = {a0.x * w0 + b0.x * w1, a0.y * w0 + b0.y * w1, a0.z * w0 + b0.z * w1, a0.w * w0 + b0.w * w1,
                      a1.x * w0 + b1.x * w1, a1.y * w0 + b1.y * w1, a1.z * w0 + b1.z * w1, a1.w * w0 + b1.w * w1};
  __nv_bfloat16* dst = out + (int64_t)t.head * out_stride_h + row * out_stride_t;
  if (out_stride_d <= 1) {
    uint4 u;
    u.x = pack_bf16x2(v[0], v[1]);
    u.y = pack_bf16x2(v[2], v[3]);
    u.z = pack_bf16x2(v[4], v[5]);
    u.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4*>(dst + c) = u;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) dst[(int64_t)(c + e) * out_stride_d] = __float2bfloat16_rn(v[e]);
  }
  if (c == 0 && lse) lse[li] = nl;
}

}  // namespace

int launch_merge(float* out, float* lse, const void* block_out, int32_t block_out_is_f32, const float* block_lse,
                 float* weight_out, int64_t seqlen, int32_t heads, int32_t head_dim, cudaStream_t stream) {
  const int64_t rows = seqlen * heads;
  if (rows == 0) return 0;
  const int64_t blocks = (rows * (head_dim / 8) + 255) / 256;
  if (head_dim == 128) {
    if (block_out_is_f32)
      merge_kernel<128, false><<<blocks, 256, 0, stream>>>(out, lse, block_out, block_lse, weight_out, seqlen, heads);
    else
      merge_kernel<128, true><<<blocks, 256, 0, stream>>>(out, lse, block_out, block_lse, weight_out, seqlen, heads);
  } else if (head_dim == 64) {
    if (block_out_is_f32)
      merge_kernel<64, false><<<blocks, 256, 0, stream>>>(out, lse, block_out, block_lse, weight_out, seqlen, heads);
    else
      merge_kernel<64, true><<<blocks, 256, 0, stream>>>(out, lse, block_out, block_lse, weight_out, seqlen, heads);
  } else {
    return (int)cudaErrorInvalidValue;
  }
  return launched();
}

int launch_merge_halves(const TileTask* tasks, int ntasks, const float* part, const float* part_lse, int heads,
                        int64_t q_len, int head_dim, void* out, int64_t out_stride_h, int64_t out_stride_t,
                        int64_t out_stride_d, float* lse, cudaStream_t stream) {
  if (ntasks <= 0) return 0;
  const int64_t part_stride = (int64_t)heads * q_len * head_dim, lse_part_stride = (int64_t)heads * q_len;
  auto o = static_cast<__nv_bfloat16*>(out);
  if (head_dim == 128) {
    merge_halves_kernel<128><<<dim3((unsigned)ntasks, 256 / 16), 256, 0, stream>>>(
        tasks, part, part_lse, part_stride, lse_part_stride, q_len, o, out_stride_h, out_stride_t, out_stride_d, lse);
  } else if (head_dim == 64) {
    merge_halves_kernel<64><<<dim3((unsigned)ntasks, 256 / 32), 256, 0, stream>>>(
        tasks, part, part_lse, part_stride, lse_part_stride, q_len, o, out_stride_h, out_stride_t, out_stride_d, lse);
  } else {
    return (int)cudaErrorInvalidValue;
  }
  return launched();
}

int launch_bwd_preprocess(const void* dout, const void* out, const float* lse, int64_t total, int64_t t_pad,
                          int32_t heads, int32_t head_dim, float* rows, float* dq_f32_zero, void* dq_other_zero,
                          size_t other_bytes, cudaStream_t stream) {
  const int64_t n = total * heads;
  if (n == 0) return 0;
  if (dq_other_zero) {
    cudaError_t e = cudaMemsetAsync(dq_other_zero, 0, other_bytes, stream);
    if (e != cudaSuccess) return (int)e;
  }
  const int64_t blocks = (n * (head_dim / 8) + 255) / 256;
  auto d = reinterpret_cast<const __nv_bfloat16*>(dout);
  auto o = reinterpret_cast<const __nv_bfloat16*>(out);
  float2* r2 = reinterpret_cast<float2*>(rows);
  if (head_dim == 128) delta_kernel<128><<<blocks, 256, 0, stream>>>(d, o, lse, r2, dq_f32_zero, total, t_pad, heads);
  else if (head_dim == 64) delta_kernel<64><<<blocks, 256, 0, stream>>>(d, o, lse, r2, dq_f32_zero, total, t_pad, heads);
  else return (int)cudaErrorInvalidValue;
  return launched();
}

int launch_fixed_to_bf16(const unsigned long long* src, void* dst, int64_t T, int H, int D, cudaStream_t stream) {
  const int64_t n2 = T * H * D / 2;
  if (n2 == 0) return 0;
  const int64_t blocks = std::min<int64_t>((n2 + 255) / 256, 148 * 16);
  fixed_to_bf16_kernel<<<blocks, 256, 0, stream>>>(src, reinterpret_cast<__nv_bfloat162*>(dst), T, H, D,
                                                   fixed_tpad(T));
  return launched();
}

int launch_fixed_add_f32(const unsigned long long* src, float* dst, int64_t T, int H, int D, cudaStream_t stream) {
  const int64_t n2 = T * H * D / 2;
  if (n2 == 0) return 0;
  const int64_t blocks = std::min<int64_t>((n2 + 255) / 256, 148 * 16);
  fixed_add_f32_kernel<<<blocks, 256, 0, stream>>>(src, reinterpret_cast<float2*>(dst), T, H, D, fixed_tpad(T));
  return launched();
}

int launch_convert_bf16_transposed(const float* src, void* dst, int H, int64_t S, int D, cudaStream_t stream) {
  if ((int64_t)H * S == 0) return 0;
  const dim3 grid((unsigned)((S + 31) / 32), (unsigned)(D / 32), (unsigned)H);
  transpose_bf16_kernel<<<grid, dim3(32, 8), 0, stream>>>(src, static_cast<__nv_bfloat16*>(dst), S, D);
  return launched();
}

namespace {
thread_local size_t g_launches = 0;
thread_local cudaEvent_t g_ev_start = nullptr, g_ev_stop = nullptr;
}

void set_kernel_events(cudaEvent_t start, cudaEvent_t stop) {
  g_ev_start = start;
  g_ev_stop = stop;
}

int kernel_event_start(cudaStream_t stream) { return g_ev_start ? (int)cudaEventRecord(g_ev_start, stream) : 0; }

int kernel_event_stop(cudaStream_t stream) { return g_ev_stop ? (int)cudaEventRecord(g_ev_stop, stream) : 0; }

int launched() {
  ++g_launches;
  return (int)cudaGetLastError();
}

size_t launch_count() { return g_launches; }

int launch_inline_copy(void* dst, const void* src, size_t bytes, cudaStream_t stream) {
  InlineChunk c;
  const unsigned char* p = static_cast<const unsigned char*>(src);
  for (size_t off = 0; off < bytes; off += kInlineBytes) {
    const size_t n = std::min<size_t>(kInlineBytes, bytes - off);
    c.dst = reinterpret_cast<uint4*>(static_cast<unsigned char*>(dst) + off);
    c.n16 = (uint32_t)((n + 15) / 16);
    c.pad = 0;
    memset(c.data, 0, (size_t)c.n16 * 16);
    memcpy(c.data, p + off, n);
    inline_copy_kernel<<<1, 256, 0, stream>>>(c);
    const int e = launched();
    if (e) return e;
  }
  return 0;
}

int launch_schedule(void* image_dst, const void* image, size_t bytes, size_t off_tiles, int ngroups, TileTask* tasks,
                    int ntasks, int* status, cudaStream_t stream, bool* status_cleared) {
  *status_cleared = false;
  if (ntasks == 0 || ngroups == 0) return 0;
  if (bytes > (size_t)kInlineBytes || bytes % 16) {  // larger images: copy in pieces, then expand
    int e = launch_inline_copy(image_dst, image, bytes, stream);
    if (e) return e;
    return launch_expand_tasks(static_cast<const PlanGroup*>(image_dst), ngroups,
                               reinterpret_cast<const TileTask*>(static_cast<unsigned char*>(image_dst) + off_tiles),
                               tasks, ntasks, stream);
  }
  *status_cleared = status != nullptr;
  if (bytes <= 2048) return launch_schedule_t<2048>(image_dst, image, bytes, off_tiles, ngroups, tasks, ntasks, status, stream);
  if (bytes <= 8192) return launch_schedule_t<8192>(image_dst, image, bytes, off_tiles, ngroups, tasks, ntasks, status, stream);
  return launch_schedule_t<kInlineBytes>(image_dst, image, bytes, off_tiles, ngroups, tasks, ntasks, status, stream);
}

int launch_expand_tasks(const PlanGroup* groups, int ngroups, const TileTask* tiles, TileTask* tasks, int ntasks,
                        cudaStream_t stream) {
  if (ntasks == 0 || ngroups == 0) return 0;
  const int blocks = std::min((ntasks + 255) / 256, 148 * 4);
  expand_tasks_kernel<<<blocks, 256, 0, stream>>>(groups, ngroups, tiles, tasks, ntasks);
  return launched();
}

namespace {
// dst [B][A][row] = src [A][B][row]: the exchange of the leading two axes of an array of rows
template <typename U>
__global__ void __launch_bounds__(256) swap01_kernel(const U* __restrict__ src, U* __restrict__ dst, int64_t A,
                                                     int64_t B, int64_t units) {
  const int64_t n = A * B * units;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t u = i % units, ab = i / units;
    const int64_t a = ab / B, b = ab % B;
    dst[(b * A + a) * units + u] = src[i];
  }
}
}  // namespace

int launch_swap01(const void* src, void* dst, int64_t A, int64_t B, int64_t row_bytes, cudaStream_t stream) {
  if (A * B * row_bytes == 0) return 0;
  const bool v16 = row_bytes % 16 == 0 && reinterpret_cast<uintptr_t>(src) % 16 == 0 &&
                   reinterpret_cast<uintptr_t>(dst) % 16 == 0;
  const int64_t units = row_bytes / (v16 ? 16 : 4);
  const int64_t blocks = std::min<int64_t>((A * B * units + 255) / 256, 148 * 16);
  if (v16)
    swap01_kernel<uint4><<<blocks, 256, 0, stream>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), A, B,
                                                     units);
  else
    swap01_kernel<uint32_t><<<blocks, 256, 0, stream>>>(static_cast<const uint32_t*>(src),
                                                        static_cast<uint32_t*>(dst), A, B, units);
  return launched();
}

int launch_convert_bf16(const float* src, void* dst, int64_t n, float mul, cudaStream_t stream) {
  if (n == 0) return 0;
  const int64_t n4 = n / 4;  // n is a multiple of the head dim (64 or 128)
  const int64_t blocks = std::min<int64_t>((n4 + 255) / 256, 148 * 16);
  convert_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<const float4*>(src), reinterpret_cast<uint2*>(dst), n4,
                                             mul);
  return launched();
}

}  // namespace cbv
