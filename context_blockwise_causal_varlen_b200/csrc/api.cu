// The C ABI of libcbv.so (include/cbv.h): argument checks, workspace layout,
// tensor-map encoding and the launch sequence of every call.
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/cbv.h"
#include "api_internal.h"
#include "kernels.h"
#include "plan.h"
#include "ptx.cuh"

using namespace cbv;

namespace {

thread_local std::string g_err;

// An NVTX range around one call (visible to a profiler; close to free without one attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int cuda_fail(int err, const char* what) {
  return fail(CBV_ERR_CUDA, "%s: %s", what, cudaGetErrorString((cudaError_t)err));
}

constexpr size_t kAlign = 256;
constexpr int32_t kPairRows = 256;  // q rows per forward task: two 128-row tiles
constexpr size_t kStatusBytes = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Bump allocator over the caller's workspace.
struct Carve {
  char* base;
  size_t off = 0;
  explicit Carve(void* b) : base(static_cast<char*>(b)) {}
  void* take(size_t bytes) {
    void* p = base ? base + off : nullptr;
    off += align_up(bytes);
    return p;
  }
};

// Resolved once, thread-safely (a function-local static), on the first call from any thread.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    cudaDriverEntryPointQueryResult q;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
  }();
  return fn;
}

// rank-n tiled map; dims/strides in elements (strides for dims 1..n-1)
int make_map(CUtensorMap* m, CUtensorMapDataType dt, int esize, int rank, const void* ptr, const uint64_t* dims,
             const uint64_t* strides_el, const uint32_t* box, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return fail(CBV_ERR_CUDA, "cuTensorMapEncodeTiled is not available (driver too old or no GPU)");
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_el[i] * esize;
  CUresult r = fn(m, dt, rank, const_cast<void*>(ptr), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CBV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return CBV_OK;
}

// token-major bf16 [T, H, D] (or any strides) as (D, H, T), box (64, 1, rows)
int map_thd(CUtensorMap* m, const void* ptr, int64_t T, int H, int D, int64_t stride_t, int64_t stride_h, int rows) {
  uint64_t dims[3] = {(uint64_t)D, (uint64_t)H, (uint64_t)std::max<int64_t>(T, 1)};
  uint64_t st[2] = {(uint64_t)stride_h, (uint64_t)stride_t};
  uint32_t box[3] = {64, 1, (uint32_t)rows};
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 3, ptr, dims, st, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

float resolve_scale(float scale, int D) { return scale > 0.f ? scale : 1.0f / std::sqrt((float)D); }
constexpr float kLog2e = 1.4426950408889634f;

int check_header(uint32_t size, uint32_t expect, uint32_t ver) {
  if (ver != CBV_ABI_VERSION) return fail(CBV_ERR_VERSION, "abi_version %u, library is %d", ver, CBV_ABI_VERSION);
  if (size != expect) return fail(CBV_ERR_VERSION, "struct_size %u, library expects %u", size, expect);
  return CBV_OK;
}

int check_heads(int H, int Hkv, int D) {
  if (D != 64 && D != 128) return fail(CBV_ERR_UNSUPPORTED_HEAD_DIM, "head_dim %d (supported: 64, 128)", D);
  if (H <= 0 || Hkv <= 0) return fail(CBV_ERR_BAD_SHAPE, "num_heads and num_kv_heads must be positive");
  if (H % Hkv) return fail(CBV_ERR_GQA_MISMATCH, "GQA mismatch: %d q heads vs %d kv heads", H, Hkv);
  return CBV_OK;
}

int check_cu(const int32_t* cu, int32_t num_docs, int64_t total, const char* what) {
  std::string e = check_cu_seqlens(cu, num_docs);
  if (!e.empty()) return fail(CBV_ERR_BAD_CU_SEQLENS, "%s: %s", what, e.c_str());
  if ((int64_t)cu[num_docs] > total)
    return fail(CBV_ERR_BAD_CU_SEQLENS, "%s: last offset %d exceeds the %lld rows", what, cu[num_docs], (long long)total);
  return CBV_OK;
}

int check_max_seqlen(const int32_t* cu, int32_t num_docs, int32_t max_seqlen) {
  if (max_seqlen <= 0) return CBV_OK;
  for (int d = 0; d < num_docs; ++d)
    if (cu[d + 1] - cu[d] > max_seqlen)
      return fail(CBV_ERR_BAD_ARG, "max_seqlen %d is below document %d's length %d", max_seqlen, d, cu[d + 1] - cu[d]);
  return CBV_OK;
}

int zero_status(void* ws, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(ws, 0, kStatusBytes, s);
  return e == cudaSuccess ? CBV_OK : cuda_fail(e, "clearing the status word");
}

// A schedule in the workspace: the expanded task list (written on the device) and one image of
// groups | tiles | segs (uploaded), each part 16-byte aligned.
struct PlanDev {
  TileTask* tasks = nullptr;
  Seg* segs = nullptr;
  PlanGroup* groups = nullptr;
  TileTask* tiles = nullptr;
  unsigned char* image = nullptr;
  size_t off_tiles = 0, off_segs = 0, image_bytes = 0;
};

size_t up16(size_t x) { return (x + 15) / 16 * 16; }

PlanDev carve_plan(Carve& c, const Plan& p) {
  PlanDev d;
  d.tasks = static_cast<TileTask*>(c.take(std::max<size_t>(1, p.tasks.size()) * sizeof(TileTask)));
  d.off_tiles = up16(p.groups.size() * sizeof(PlanGroup));
  d.off_segs = d.off_tiles + up16(p.tiles.size() * sizeof(TileTask));
  d.image_bytes = d.off_segs + up16(p.segs.size() * sizeof(Seg));
  d.image = static_cast<unsigned char*>(c.take(std::max<size_t>(16, d.image_bytes)));
  if (d.image) {
    d.groups = reinterpret_cast<PlanGroup*>(d.image);
    d.tiles = reinterpret_cast<TileTask*>(d.image + d.off_tiles);
    d.segs = reinterpret_cast<Seg*>(d.image + d.off_segs);
  }
  return d;
}

// Uploads the compact schedule inside kernel launch parameters (no copy engine, no host wait)
// and expands the task list on the device.  With `status`, the call's status word is cleared
// too: by the schedule launch itself when it is a single one, else by a memset.
int upload_plan(const PlanDev& d, const Plan& p, cudaStream_t s, int* status = nullptr) {
  bool cleared = false;
  if (!p.tasks.empty()) {
    std::vector<unsigned char> img(d.image_bytes, 0);
    memcpy(img.data(), p.groups.data(), p.groups.size() * sizeof(PlanGroup));
    memcpy(img.data() + d.off_tiles, p.tiles.data(), p.tiles.size() * sizeof(TileTask));
    memcpy(img.data() + d.off_segs, p.segs.data(), p.segs.size() * sizeof(Seg));
    const int e = launch_schedule(d.image, img.data(), img.size(), d.off_tiles, (int)p.groups.size(), d.tasks,
                                  (int)p.tasks.size(), status, s, &cleared);
    if (e) return cuda_fail(e, "uploading the schedule");
  }
  return status && !cleared ? zero_status(status, s) : CBV_OK;
}

int launch_rc(int e, const char* what) { return e == 0 ? CBV_OK : cuda_fail(e, what); }

// Streaming multiprocessors of the current device (0 if it cannot be asked).
int sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return sms;
}

int grid_of(size_t tasks, int heads) {
  const size_t g = tasks * (size_t)heads;
  return g > (size_t)INT32_MAX ? -1 : (int)g;
}

// ------------------------------------------------------------------------ ring forward
int ring_common_checks(const cbv_ring_args* a) {
  if (!a) return fail(CBV_ERR_BAD_ARG, "args is NULL");
  int rc = check_header(a->struct_size, sizeof(cbv_ring_args), a->abi_version);
  if (rc) return rc;
  if ((rc = check_heads(a->num_heads, a->num_kv_heads, a->head_dim))) return rc;
  if (!a->causal) return fail(CBV_ERR_NOT_CAUSAL, "the ring layouts are causal only (zig-zag is meaningless otherwise)");
  if (a->cp < 1) return fail(CBV_ERR_BAD_ARG, "cp must be >= 1");
  if (a->layout != CBV_LAYOUT_ZIGZAG && a->layout != CBV_LAYOUT_CONTIGUOUS) return fail(CBV_ERR_BAD_ARG, "bad layout");
  if ((rc = check_cu(a->cu_seqlens, a->num_docs, a->total, "cu_seqlens"))) return rc;
  if (a->cu_seqlens[a->num_docs] != a->total)
    return fail(CBV_ERR_BAD_CU_SEQLENS, "cu_seqlens must end at total (%lld)", (long long)a->total);
  if ((rc = check_max_seqlen(a->cu_seqlens, a->num_docs, a->max_seqlen))) return rc;
  std::string e = check_divisible(a->cu_seqlens, a->num_docs, a->cp, (Layout)a->layout);
  if (!e.empty()) return fail(CBV_ERR_NOT_DIVISIBLE_2CP, "%s", e.c_str());
  if (a->schedule != CBV_SCHEDULE_FUSED && a->schedule != CBV_SCHEDULE_STEPWISE)
    return fail(CBV_ERR_BAD_ARG, "bad schedule");
  return CBV_OK;
}

RingFwdLayout ring_fwd_layout(const cbv_ring_args* a) {
  RingFwdLayout L;
  Carve c(nullptr);
  c.take(kStatusBytes);
  if (a->schedule == CBV_SCHEDULE_FUSED) {
    L.fused = plan_ring_fwd(a->cu_seqlens, a->num_docs, a->cp, (Layout)a->layout, a->window, a->num_heads, -1,
                            kPairRows, true);
    carve_plan(c, L.fused);
  } else {
    for (int s = 0; s < a->cp; ++s) {
      L.steps.push_back(
          plan_ring_fwd(a->cu_seqlens, a->num_docs, a->cp, (Layout)a->layout, a->window, a->num_heads, s, kPairRows,
                        false));
      carve_plan(c, L.steps.back());
    }
    c.take((size_t)a->total * a->num_heads * a->head_dim * sizeof(float));  // running out (fp32)
  }
  L.bytes = c.off;
  return L;
}

FwdParams ring_fwd_params(const cbv_ring_args* a, int* rc) {
  FwdParams p{};
  const int D = a->head_dim, H = a->num_heads, Hkv = a->num_kv_heads;
  *rc = map_thd(&p.tm_q, a->q, a->total, H, D, (int64_t)H * D, D, 128);
  if (!*rc) *rc = map_thd(&p.tm_k, a->k, a->total, Hkv, D, (int64_t)Hkv * D, D, 128);
  if (!*rc) *rc = map_thd(&p.tm_v, a->v, a->total, Hkv, D, (int64_t)Hkv * D, D, 128);
  p.num_heads = H;
  p.heads_per_kv = H / Hkv;
  p.scale_log2 = resolve_scale(a->scale, D) * kLog2e;
  p.window = a->window > 0 ? a->window : 0;
  p.out_stride_t = (int64_t)H * D;
  p.out_stride_h = D;
  p.lse = a->lse;
  p.lse_stride_h = a->total;
  p.lse_stride_t = 1;
  p.block_size = 1;
  p.q_rows = p.kv_rows = a->total;
  return p;
}

}  // namespace

namespace cbv {
void set_last_error(const char* msg) { g_err = msg; }
}  // namespace cbv

extern "C" {

const char* cbv_last_error_message(void) { return g_err.c_str(); }
int cbv_abi_version(void) { return CBV_ABI_VERSION; }

size_t cbv_launch_count(void) { return cbv::launch_count(); }

int cbv_set_kernel_events(void* start_event, void* stop_event) {
  cbv::set_kernel_events(static_cast<cudaEvent_t>(start_event), static_cast<cudaEvent_t>(stop_event));
  return CBV_OK;
}

int cbv_build_flags(void) {
#ifdef CBV_DEBUG
  return CBV_BUILD_DEBUG;
#else
  return 0;
#endif
}

int cbv_read_status(const void* workspace, int* status_out, void* stream) {
  if (!workspace || !status_out) return fail(CBV_ERR_BAD_ARG, "NULL argument");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
  *status_out = v;
  if (v != 0) return fail(CBV_ERR_TIMEOUT, "a kernel gave up a wait (code 0x%x)", v);
  return CBV_OK;
}

// ------------------------------------------------------------------------ planner exports
int cbv_local_cu_seqlens(const int32_t* cu, int32_t num_docs, int32_t cp, int32_t layout, int32_t* out) {
  if (!out) return fail(CBV_ERR_BAD_ARG, "out is NULL");
  std::string e = check_cu_seqlens(cu, num_docs);
  if (!e.empty()) return fail(CBV_ERR_BAD_CU_SEQLENS, "%s", e.c_str());
  e = check_divisible(cu, num_docs, cp, (Layout)layout);
  if (!e.empty()) return fail(CBV_ERR_NOT_DIVISIBLE_2CP, "%s", e.c_str());
  local_cu_seqlens(cu, num_docs, cp, out);
  return CBV_OK;
}

int cbv_half_cu_seqlens(const int32_t* cu, int32_t num_docs, int32_t cp, int32_t* out) {
  if (!out) return fail(CBV_ERR_BAD_ARG, "out is NULL");
  std::string e = check_cu_seqlens(cu, num_docs);
  if (!e.empty()) return fail(CBV_ERR_BAD_CU_SEQLENS, "%s", e.c_str());
  e = check_divisible(cu, num_docs, cp, kZigZag);
  if (!e.empty()) return fail(CBV_ERR_NOT_DIVISIBLE_2CP, "%s", e.c_str());
  half_cu_seqlens(cu, num_docs, cp, out);
  return CBV_OK;
}

int cbv_get_half_index(const int32_t* cu_local, int32_t num_docs, int32_t front, int32_t* idx_out, int64_t* count_out) {
  std::string e = check_cu_seqlens(cu_local, num_docs);
  if (!e.empty()) return fail(CBV_ERR_BAD_CU_SEQLENS, "%s", e.c_str());
  for (int d = 0; d < num_docs; ++d)
    if ((cu_local[d + 1] - cu_local[d]) % 2) return fail(CBV_ERR_NOT_DIVISIBLE_2CP, "local document %d has odd length", d);
  const int64_t n = get_half_index(cu_local, num_docs, front != 0, idx_out);
  if (count_out) *count_out = n;
  return CBV_OK;
}

int cbv_get_half_lse(const float* lse, int32_t num_heads, const int32_t* cu_local, int32_t num_docs, int32_t front,
                     float* out) {
  if (!lse || !out || num_heads < 0) return fail(CBV_ERR_BAD_ARG, "bad argument");
  int64_t n = 0;
  int rc = cbv_get_half_index(cu_local, num_docs, front, nullptr, &n);
  if (rc) return rc;
  std::vector<int32_t> idx(n);
  get_half_index(cu_local, num_docs, front != 0, idx.data());
  const int64_t S = cu_local[num_docs];
  for (int h = 0; h < num_heads; ++h)
    for (int64_t i = 0; i < n; ++i) out[h * n + i] = lse[h * S + idx[i]];
  return CBV_OK;
}

int cbv_rank_tokens(const int32_t* cu, int32_t num_docs, int32_t cp, int32_t rank, int32_t layout, int32_t* out) {
  if (!out || rank < 0 || rank >= cp) return fail(CBV_ERR_BAD_ARG, "bad rank or NULL out");
  std::string e = check_cu_seqlens(cu, num_docs);
  if (!e.empty()) return fail(CBV_ERR_BAD_CU_SEQLENS, "%s", e.c_str());
  e = check_divisible(cu, num_docs, cp, (Layout)layout);
  if (!e.empty()) return fail(CBV_ERR_NOT_DIVISIBLE_2CP, "%s", e.c_str());
  rank_tokens(cu, num_docs, cp, rank, (Layout)layout, out);
  return CBV_OK;
}

int cbv_rank_pair_counts(const int32_t* cu, int32_t num_docs, int32_t cp, int32_t layout, int32_t window,
                         int64_t* counts_out) {
  if (!counts_out) return fail(CBV_ERR_BAD_ARG, "counts_out is NULL");
  std::string e = check_cu_seqlens(cu, num_docs);
  if (!e.empty()) return fail(CBV_ERR_BAD_CU_SEQLENS, "%s", e.c_str());
  e = check_divisible(cu, num_docs, cp, (Layout)layout);
  if (!e.empty()) return fail(CBV_ERR_NOT_DIVISIBLE_2CP, "%s", e.c_str());
  rank_pair_counts(cu, num_docs, cp, (Layout)layout, window, counts_out);
  return CBV_OK;
}

int cbv_ring_step(int32_t rank, int32_t step, int32_t cp, int32_t layout, int32_t* src_out, int32_t* kind_out) {
  if (!src_out || !kind_out || cp < 1 || rank < 0 || rank >= cp || step < 0 || step >= cp)
    return fail(CBV_ERR_BAD_ARG, "bad argument");
  ring_step(rank, step, cp, (Layout)layout, src_out, kind_out);
  return CBV_OK;
}

int cbv_plan_zigzag(const int32_t* cu, int32_t num_docs, int32_t cp, int32_t layout, cbv_ring_block* blocks,
                    int32_t max_blocks, int32_t* num_blocks_out, cbv_row_run* runs, int32_t max_runs,
                    int32_t* num_runs_out) {
  if (!num_blocks_out || !num_runs_out) return fail(CBV_ERR_BAD_ARG, "NULL count");
  if (layout != CBV_LAYOUT_ZIGZAG && layout != CBV_LAYOUT_CONTIGUOUS) return fail(CBV_ERR_BAD_ARG, "bad layout");
  std::string e = check_cu_seqlens(cu, num_docs);
  if (!e.empty()) return fail(CBV_ERR_BAD_CU_SEQLENS, "%s", e.c_str());
  e = check_divisible(cu, num_docs, cp, (Layout)layout);
  if (!e.empty()) return fail(CBV_ERR_NOT_DIVISIBLE_2CP, "%s", e.c_str());
  std::vector<RingBlock> bl;
  std::vector<RowRun> rr;
  ring_blocks(cu, num_docs, cp, (Layout)layout, &bl, &rr);
  *num_blocks_out = (int32_t)bl.size();
  *num_runs_out = (int32_t)rr.size();
  if (!blocks || !runs) return CBV_OK;
  if (max_blocks < (int32_t)bl.size() || max_runs < (int32_t)rr.size())
    return fail(CBV_ERR_BAD_ARG, "capacity too small: %zu blocks and %zu runs", bl.size(), rr.size());
  static_assert(sizeof(cbv_ring_block) == sizeof(RingBlock) && sizeof(cbv_row_run) == sizeof(RowRun), "layouts");
  for (size_t i = 0; i < bl.size(); ++i) {
    const RingBlock& b = bl[i];
    blocks[i] = cbv_ring_block{b.rank, b.step, b.src, b.kind, b.causal, b.q_half, b.k_half,
                               b.q_run0, b.q_nruns, b.k_run0, b.k_nruns};
  }
  for (size_t i = 0; i < rr.size(); ++i) runs[i] = cbv_row_run{rr[i].doc, rr[i].row0, rr[i].rows, rr[i].pos0, rr[i].local0};
  return CBV_OK;
}

// ------------------------------------------------------------------------ block forward
static int block_fwd_checks(const cbv_block_fwd_args* a) {
  if (!a) return fail(CBV_ERR_BAD_ARG, "args is NULL");
  int rc = check_header(a->struct_size, sizeof(cbv_block_fwd_args), a->abi_version);
  if (rc) return rc;
  if ((rc = check_heads(a->num_heads, a->num_kv_heads, a->head_dim))) return rc;
  if ((rc = check_cu(a->cu_seqlens_q, a->num_docs, a->total_q, "cu_seqlens_q"))) return rc;
  if ((rc = check_cu(a->cu_seqlens_k, a->num_docs, a->total_k, "cu_seqlens_k"))) return rc;
  if ((rc = check_max_seqlen(a->cu_seqlens_q, a->num_docs, a->max_seqlen))) return rc;
  if ((rc = check_max_seqlen(a->cu_seqlens_k, a->num_docs, a->max_seqlen))) return rc;
  if (a->merge && a->out_dtype != CBV_DTYPE_F32) return fail(CBV_ERR_BAD_DTYPE, "merge = 1 needs an f32 out");
  if (a->out_dtype != CBV_DTYPE_F32 && a->out_dtype != CBV_DTYPE_BF16) return fail(CBV_ERR_BAD_DTYPE, "bad out_dtype");
  return CBV_OK;
}

size_t cbv_block_fwd_workspace_size(const cbv_block_fwd_args* a) {
  if (block_fwd_checks(a)) return 0;
  Plan p = plan_block_fwd(a->cu_seqlens_q, a->cu_seqlens_k, a->q_pos_base, a->k_pos_base, a->num_docs, a->causal != 0,
                          a->window, a->num_heads, kPairRows);
  Carve c(nullptr);
  c.take(kStatusBytes);
  carve_plan(c, p);
  return c.off;
}

int cbv_attn_block_fwd(const cbv_block_fwd_args* a, void* stream) {
  NvtxRange nvtx_range("cbv_attn_block_fwd");
  int rc = block_fwd_checks(a);
  if (rc) return rc;
  if (a->total_q == 0) return CBV_OK;  // no query rows: nothing to write
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = a->head_dim, H = a->num_heads, Hkv = a->num_kv_heads;
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->out))
    return fail(CBV_ERR_MISALIGNED, "tensors must be 16-byte aligned");
  // without key rows no k tile is ever loaded; the maps then describe one q row instead
  const void* kp = a->total_k > 0 ? a->k : a->q;
  const void* vp = a->total_k > 0 ? a->v : a->q;
  const int64_t kst = a->total_k > 0 ? (int64_t)Hkv * D : (int64_t)H * D;
  Plan plan = plan_block_fwd(a->cu_seqlens_q, a->cu_seqlens_k, a->q_pos_base, a->k_pos_base, a->num_docs,
                             a->causal != 0, a->window, H, kPairRows);
  Carve c(a->workspace);
  int* status = static_cast<int*>(c.take(kStatusBytes));
  PlanDev pd = carve_plan(c, plan);
  if (!a->workspace || a->workspace_bytes < c.off)
    return fail(CBV_ERR_WORKSPACE_TOO_SMALL, "workspace needs %zu bytes", c.off);
  FwdParams p{};
  if ((rc = map_thd(&p.tm_q, a->q, a->total_q, H, D, (int64_t)H * D, D, 128))) return rc;
  if ((rc = map_thd(&p.tm_k, kp, a->total_k, Hkv, D, kst, D, 128))) return rc;
  if ((rc = map_thd(&p.tm_v, vp, a->total_k, Hkv, D, kst, D, 128))) return rc;
  p.tasks = pd.tasks;
  p.segs = pd.segs;
  p.num_tasks = (int)plan.tasks.size();
  p.num_heads = H;
  p.heads_per_kv = H / Hkv;
  p.scale_log2 = resolve_scale(a->scale, D) * kLog2e;
  p.window = a->window > 0 ? a->window : 0;
  p.out = a->out;
  p.out_stride_t = (int64_t)H * D;
  p.out_stride_h = D;
  p.lse = a->lse;
  p.lse_stride_h = a->total_q;
  p.lse_stride_t = 1;
  p.out_mode = a->merge ? kOutMerge : (a->out_dtype == CBV_DTYPE_F32 ? kOutF32 : kOutBf16);
  p.block_size = 1;
  p.q_rows = a->total_q;
  p.kv_rows = a->total_k > 0 ? a->total_k : a->total_q;  // without keys the maps describe q
  p.status = status;
  if ((rc = upload_plan(pd, plan, s, status))) return rc;
  const int grid = grid_of(plan.tasks.size(), 1);
  if (grid < 0) return fail(CBV_ERR_BAD_SHAPE, "too many tiles");
  return launch_rc(launch_fwd_pingpong(p, D, false, grid, s), "block forward launch");
}

// ------------------------------------------------------------------------ merge
int cbv_attn_merge(float* out, float* lse, const void* block_out, int32_t block_out_dtype, const float* block_lse,
                   float* weight_out, int64_t seqlen, int32_t num_heads, int32_t head_dim, void* stream) {
  NvtxRange nvtx_range("cbv_attn_merge");
  if (head_dim != 64 && head_dim != 128) return fail(CBV_ERR_UNSUPPORTED_HEAD_DIM, "head_dim %d", head_dim);
  if (seqlen < 0 || num_heads <= 0) return fail(CBV_ERR_BAD_SHAPE, "bad shape");
  if (seqlen == 0) return CBV_OK;
  if (!out || !lse || !block_out || !block_lse) return fail(CBV_ERR_BAD_ARG, "NULL tensor");
  if (block_out_dtype != CBV_DTYPE_BF16 && block_out_dtype != CBV_DTYPE_F32) return fail(CBV_ERR_BAD_DTYPE, "bad dtype");
  if (!aligned16(out) || !aligned16(block_out)) return fail(CBV_ERR_MISALIGNED, "tensors must be 16-byte aligned");
  return launch_rc(launch_merge(out, lse, block_out, block_out_dtype == CBV_DTYPE_F32, block_lse, weight_out, seqlen,
                                num_heads, head_dim, static_cast<cudaStream_t>(stream)),
                   "merge launch");
}

// ------------------------------------------------------------------------ ring forward
size_t cbv_zigzag_ring_fwd_workspace_size(const cbv_ring_args* a) {
  if (ring_common_checks(a)) return 0;
  return ring_fwd_layout(a).bytes;
}

int cbv_debug_ring_fwd_stalled(const cbv_ring_args* a, uint64_t wait_limit_ns, void* stream) {
  NvtxRange nvtx_range("cbv_debug_ring_fwd_stalled");
  if (wait_limit_ns < 100000ull || wait_limit_ns > 1000000000ull)
    return fail(CBV_ERR_BAD_ARG, "wait_limit_ns must be in [1e5, 1e9]");
  if (a && a->schedule != CBV_SCHEDULE_FUSED) return fail(CBV_ERR_BAD_ARG, "the fused schedule only");
  RingFwdLayout L;
  int rc = cbv::ring_fwd_plan(a, &L);
  if (rc || a->total == 0) return rc;
  if (!a->workspace || a->workspace_bytes < L.bytes)
    return fail(CBV_ERR_WORKSPACE_TOO_SMALL, "workspace needs %zu bytes", L.bytes);
  return cbv::ring_fwd_run(a, L, a->workspace, static_cast<cudaStream_t>(stream), wait_limit_ns, 1);
}

int cbv_zigzag_ring_fwd(const cbv_ring_args* a, void* stream) {
  NvtxRange nvtx_range("cbv_zigzag_ring_fwd");
  RingFwdLayout L;
  int rc = cbv::ring_fwd_plan(a, &L);
  if (rc || a->total == 0) return rc;  // no rows: nothing to write
  if (!a->workspace || a->workspace_bytes < L.bytes)
    return fail(CBV_ERR_WORKSPACE_TOO_SMALL, "workspace needs %zu bytes", L.bytes);
  return cbv::ring_fwd_run(a, L, a->workspace, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

int cbv::ring_fwd_plan(const cbv_ring_args* a, RingFwdLayout* L) {
  int rc = ring_common_checks(a);
  if (rc) return rc;
  if (a->total == 0) return CBV_OK;
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->out))
    return fail(CBV_ERR_MISALIGNED, "tensors must be 16-byte aligned");
  *L = ring_fwd_layout(a);
  return CBV_OK;
}

int cbv::ring_fwd_run(const cbv_ring_args* a, const RingFwdLayout& L, void* workspace, cudaStream_t s,
                      uint64_t wait_limit_ns, int withhold_loads) {
  int rc;
  Carve c(workspace);
  int* status = static_cast<int*>(c.take(kStatusBytes));
  FwdParams p = ring_fwd_params(a, &rc);
  if (rc) return rc;
  p.status = status;
  p.wait_limit_ns = wait_limit_ns;
  p.withhold_loads = withhold_loads;
  const int D = a->head_dim, H = a->num_heads;
  if (a->schedule == CBV_SCHEDULE_FUSED) {
    PlanDev pd = carve_plan(c, L.fused);
    if ((rc = upload_plan(pd, L.fused, s, status))) return rc;
    p.tasks = pd.tasks;
    p.segs = pd.segs;
    p.num_tasks = (int)L.fused.tasks.size();
    p.out = a->out;
    p.out_mode = kOutBf16;
    return launch_rc(launch_fwd_pingpong(p, D, false, grid_of(L.fused.tasks.size(), 1), s), "ring forward launch");
  }
  if ((rc = zero_status(status, s))) return rc;
  std::vector<PlanDev> pds;
  for (auto& pl : L.steps) {
    pds.push_back(carve_plan(c, pl));
    if ((rc = upload_plan(pds.back(), pl, s))) return rc;
  }
  float* acc = static_cast<float*>(c.take((size_t)a->total * H * D * sizeof(float)));
  for (int st = 0; st < a->cp; ++st) {
    char name[48];
    snprintf(name, sizeof name, "ring step %d", st);
    NvtxRange step_range(name);
    p.tasks = pds[st].tasks;
    p.segs = pds[st].segs;
    p.num_tasks = (int)L.steps[st].tasks.size();
    p.out = acc;
    p.out_mode = st == 0 ? kOutF32 : kOutMerge;
    if ((rc = launch_rc(launch_fwd_pingpong(p, D, false, grid_of(L.steps[st].tasks.size(), 1), s), "ring step launch")))
      return rc;
  }
  return launch_rc(launch_convert_bf16(acc, a->out, a->total * H * D, 1.f, s), "output conversion");
}

extern "C" {

// ------------------------------------------------------------------------ paged KV-parallel prefill
static int kvp_checks(const cbv_kvp_args* a) {
  if (!a) return fail(CBV_ERR_BAD_ARG, "args is NULL");
  int rc = check_header(a->struct_size, sizeof(cbv_kvp_args), a->abi_version);
  if (rc) return rc;
  if ((rc = check_heads(a->num_heads, a->num_kv_heads, a->head_dim))) return rc;
  if (a->q_len < 0 || a->shards < 1 || a->blocks_per_shard < 1 || a->num_blocks < 1)
    return fail(CBV_ERR_BAD_SHAPE, "bad q_len / shards / blocks");
  const int bs = a->block_size;
  if (bs < 8 || bs > 128 || 128 % bs) return fail(CBV_ERR_BAD_ARG, "block_size must be a power of two in [8, 128]");
  if (a->seg_size <= 0) return fail(CBV_ERR_BAD_ARG, "seg_size must be positive");
  if (a->kv_mode != CBV_KV_CONTIGUOUS && a->kv_mode != CBV_KV_ROUND_ROBIN) return fail(CBV_ERR_BAD_ARG, "bad kv_mode");
  if (a->global_q_offset < 0) return fail(CBV_ERR_BAD_ARG, "global_q_offset must be >= 0");
  if (!aligned16(a->q) || !aligned16(a->k_cache) || !aligned16(a->v_cache) || !aligned16(a->out))
    return fail(CBV_ERR_MISALIGNED, "tensors must be 16-byte aligned");
  if ((a->q_stride_token % 8) || (a->q_stride_head % 8)) return fail(CBV_ERR_MISALIGNED, "q strides must be multiples of 8 elements");
  if ((a->shard_out == nullptr) != (a->shard_lse == nullptr)) return fail(CBV_ERR_BAD_ARG, "shard_out and shard_lse go together");
  if (a->shard_base < 0 || a->total_shards < 0 ||
      (int64_t)a->shard_base + a->shards > (a->total_shards ? (int64_t)a->total_shards : (int64_t)a->shards))
    return fail(CBV_ERR_BAD_ARG, "shards %d from shard_base %d exceed total_shards %d", a->shards, a->shard_base,
                a->total_shards);
  return CBV_OK;
}

// Tasks of a prefill are about equal in size, so a last wave of CTAs that is at most half full
// costs as much time as a full one.  Those tail tasks run instead as two halves each, cut where
// the visible work is split evenly (TileTask::split1), so the last wave is full and half as
// long; merge_halves_kernel combines the halves' partial (out, lse).  Returns how many tasks at
// the end of the list run that way (0 without a device to ask, or when the tail is too light
// to repay the merge).
constexpr int64_t kMinSplitWork = 16 * 128;  // 16 k tiles of a 256-row task, in TileTask::work units
static int kvp_tail_tasks(const Plan& plan) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  const int nt = (int)plan.tasks.size();
  if (sms <= 0 || nt == 0) return 0;
  const int tail = nt % sms;
  if (tail == 0 || 2 * tail > sms) return 0;
  int64_t w = 0;
  for (int i = nt - tail; i < nt; ++i) w += plan.tasks[i].work;
  return w >= kMinSplitWork * tail ? tail : 0;
}

// The segment length the kernel walks: seg_size rounded up to whole 128-key tiles, so that every
// k tile starts on a page boundary.  The result does not depend on the segment length (the
// segments are merged by the online-softmax identity), only the order of the merges does.
static int32_t kvp_segment(int32_t seg_size) { return (int32_t)std::min<int64_t>(((int64_t)seg_size + 127) / 128 * 128, INT32_MAX / 2); }

static size_t kvp_layout(const cbv_kvp_args* a, Plan* plan_out, int* tail_out) {
  const int n_local = a->blocks_per_shard * a->block_size;
  Plan plan = plan_kvp(a->q_len, a->num_heads, a->shards, n_local, kvp_segment(a->seg_size), (KvMode)a->kv_mode,
                       a->block_size, a->global_q_offset, a->sliding_window, a->shard_out != nullptr, kPairRows,
                       a->shard_base, a->total_shards);
  const int tail = a->shard_out ? 0 : kvp_tail_tasks(plan);
  Carve c(nullptr);
  c.take(kStatusBytes);
  carve_plan(c, plan);
  const size_t rows = (size_t)a->num_heads * a->q_len;
  if (!a->lse || a->shard_out) c.take(rows * sizeof(float));                // lse scratch / merged lse
  if (a->shard_out) c.take(rows * a->head_dim * sizeof(float));             // merged fp32 out
  if (tail) {
    c.take(2 * rows * a->head_dim * sizeof(float));                         // the halves' partial out
    c.take(2 * rows * sizeof(float));                                       // and lse
  }
  if (plan_out) *plan_out = std::move(plan);
  if (tail_out) *tail_out = tail;
  return c.off;
}

size_t cbv_kvp_workspace_size(const cbv_kvp_args* a) {
  if (kvp_checks(a)) return 0;
  return kvp_layout(a, nullptr, nullptr);
}

int cbv_kvp_segmented_prefill(const cbv_kvp_args* a, void* stream) {
  NvtxRange nvtx_range("cbv_kvp_segmented_prefill");
  int rc = kvp_checks(a);
  if (rc) return rc;
  if (a->q_len == 0) return CBV_OK;  // no query rows: nothing to write
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Plan plan;
  int tail = 0;
  const size_t need = kvp_layout(a, &plan, &tail);
  if (!a->workspace || a->workspace_bytes < need) return fail(CBV_ERR_WORKSPACE_TOO_SMALL, "workspace needs %zu bytes", need);
  Carve c(a->workspace);
  int* status = static_cast<int*>(c.take(kStatusBytes));
  PlanDev pd = carve_plan(c, plan);
  const size_t rows = (size_t)a->num_heads * a->q_len;
  float* lse_scratch = (!a->lse || a->shard_out) ? static_cast<float*>(c.take(rows * sizeof(float))) : nullptr;
  float* acc = a->shard_out ? static_cast<float*>(c.take(rows * a->head_dim * sizeof(float))) : nullptr;
  float* part = tail ? static_cast<float*>(c.take(2 * rows * a->head_dim * sizeof(float))) : nullptr;
  float* part_lse = tail ? static_cast<float*>(c.take(2 * rows * sizeof(float))) : nullptr;
  const int D = a->head_dim, H = a->num_heads, Hkv = a->num_kv_heads, bs = a->block_size;
  FwdParams p{};
  if ((rc = map_thd(&p.tm_q, a->q, a->q_len, H, D, a->q_stride_token, a->q_stride_head, 128))) return rc;
  {
    uint64_t dims[4] = {(uint64_t)D, (uint64_t)bs, (uint64_t)Hkv, (uint64_t)a->num_blocks};
    uint64_t st[3] = {(uint64_t)D, (uint64_t)bs * D, (uint64_t)Hkv * bs * D};
    uint32_t box[4] = {64, (uint32_t)bs, 1, 1};
    if ((rc = make_map(&p.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 4, a->k_cache, dims, st, box, CU_TENSOR_MAP_SWIZZLE_128B)))
      return rc;
    if ((rc = make_map(&p.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 4, a->v_cache, dims, st, box, CU_TENSOR_MAP_SWIZZLE_128B)))
      return rc;
  }
  p.tasks = pd.tasks;
  p.segs = pd.segs;
  p.num_tasks = (int)plan.tasks.size();
  p.num_heads = H;
  p.heads_per_kv = H / Hkv;
  p.scale_log2 = resolve_scale(a->scale, D) * kLog2e;
  p.window = a->sliding_window > 0 ? a->sliding_window : 0;
  p.block_tables = a->block_tables;
  p.blocks_per_shard = a->blocks_per_shard;
  p.block_size = bs;
  p.shards = a->shards;
  p.shard_base = a->shard_base;
  p.total_shards = a->total_shards ? a->total_shards : a->shards;
  p.kv_mode = a->kv_mode;
  p.n_local = a->blocks_per_shard * bs;
  p.q_rows = a->q_len;
  p.kv_rows = a->num_blocks;  // pages of the cache
  p.status = status;
  if ((rc = upload_plan(pd, plan, s, status))) return rc;
  const int grid = grid_of(plan.tasks.size(), 1);
  if (!a->shard_out) {
    p.out = a->out;
    p.out_mode = kOutBf16;
    p.out_stride_t = a->tp_out ? 1 : D;
    p.out_stride_h = (int64_t)a->q_len * D;
    p.out_stride_d = a->tp_out ? a->q_len : 1;
    p.lse = a->lse ? a->lse : lse_scratch;
    p.lse_stride_h = a->q_len;
    p.lse_stride_t = 1;
    const int full = grid - tail;
    // the tail tasks: two CTAs each, in the same launch, so the halves take SMs as they free up
    p.split_halves = tail > 0;
    p.split_from = full;
    p.half_out = part;
    p.half_lse = part_lse;
    p.half_rows = (int64_t)rows;
    p.half_q_len = a->q_len;
    if ((rc = launch_rc(launch_fwd_pingpong(p, D, true, full + 2 * tail, s), "prefill launch"))) return rc;
    if (!tail) return CBV_OK;
    return launch_rc(launch_merge_halves(pd.tasks + full, tail, part, part_lse, H, a->q_len, D, a->out, p.out_stride_h,
                                         p.out_stride_t, p.out_stride_d, a->lse, s),
                     "prefill tail merge");
  }
  // per-shard partials, then an explicit online-softmax merge of the shards
  p.out = a->shard_out;
  p.out_mode = kOutF32;
  p.out_stride_t = D;
  p.out_stride_h = (int64_t)a->q_len * D;
  p.out_shard_stride = (int64_t)H * a->q_len * D;
  p.lse = a->shard_lse;
  p.lse_stride_h = a->q_len;
  p.lse_stride_t = 1;
  p.lse_shard_stride = (int64_t)H * a->q_len;
  if ((rc = launch_rc(launch_fwd_pingpong(p, D, true, grid, s), "prefill launch"))) return rc;
  cudaError_t e = cudaMemcpyAsync(acc, a->shard_out, rows * D * sizeof(float), cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(lse_scratch, a->shard_lse, rows * sizeof(float), cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "copying shard 0");
  for (int r = 1; r < a->shards; ++r) {
    rc = launch_rc(launch_merge(acc, lse_scratch, a->shard_out + (size_t)r * rows * D, 1, a->shard_lse + (size_t)r * rows,
                                nullptr, (int64_t)rows, 1, D, s),
                   "shard merge");
    if (rc) return rc;
  }
  if (a->lse) {
    e = cudaMemcpyAsync(a->lse, lse_scratch, rows * sizeof(float), cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "copying lse");
  }
  if (a->tp_out) return launch_rc(launch_convert_bf16_transposed(acc, a->out, H, a->q_len, D, s), "output conversion");
  return launch_rc(launch_convert_bf16(acc, a->out, (int64_t)rows * D, 1.f, s), "output conversion");
}

// ------------------------------------------------------------------------ varlen decode
size_t cbv_decode_workspace_size(const cbv_decode_args* a) {
  (void)a;
  return kStatusBytes;
}

int cbv_varlen_decode(const cbv_decode_args* a, void* stream) {
  NvtxRange nvtx_range("cbv_varlen_decode");
  if (!a) return fail(CBV_ERR_BAD_ARG, "args is NULL");
  int rc = check_header(a->struct_size, sizeof(cbv_decode_args), a->abi_version);
  if (rc) return rc;
  if ((rc = check_heads(a->num_heads, a->num_kv_heads, a->head_dim))) return rc;
  if (a->num_heads / a->num_kv_heads > 16) return fail(CBV_ERR_GQA_MISMATCH, "at most 16 q heads per kv head");
  if (a->num_seqs < 0 || a->total_q < a->num_seqs || a->total_k < 0) return fail(CBV_ERR_BAD_SHAPE, "bad sizes");
  if (a->num_seqs == 0) return CBV_OK;  // no sequences: nothing to write
  if (!a->cu_seqlens_q || !a->cu_seqlens_k) return fail(CBV_ERR_BAD_CU_SEQLENS, "cu_seqlens is NULL");
  if (!a->workspace || a->workspace_bytes < kStatusBytes) return fail(CBV_ERR_WORKSPACE_TOO_SMALL, "workspace needs %zu bytes", kStatusBytes);
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->out))
    return fail(CBV_ERR_MISALIGNED, "tensors must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (a->validate) {
    std::vector<int32_t> cq(a->num_seqs + 1), ck(a->num_seqs + 1);
    cudaError_t e = cudaMemcpyAsync(cq.data(), a->cu_seqlens_q, cq.size() * 4, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(ck.data(), a->cu_seqlens_k, ck.size() * 4, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "reading cu_seqlens");
    for (int i = 0; i < a->num_seqs; ++i)
      if (cq[i + 1] - cq[i] != 1)
        return fail(CBV_ERR_Q_LEN_NOT_ONE, "sequence %d has %d query rows (one query per sequence only)", i, cq[i + 1] - cq[i]);
    if (cq[0] < 0 || cq[a->num_seqs] > a->total_q) return fail(CBV_ERR_BAD_CU_SEQLENS, "cu_seqlens_q out of range");
    for (int i = 0; i < a->num_seqs; ++i)
      if (ck[i + 1] < ck[i]) return fail(CBV_ERR_BAD_CU_SEQLENS, "cu_seqlens_k must be non-decreasing");
    if (ck[0] < 0 || ck[a->num_seqs] > a->total_k) return fail(CBV_ERR_BAD_CU_SEQLENS, "cu_seqlens_k out of range");
  }
  const int D = a->head_dim, Hkv = a->num_kv_heads;
  DecodeParams p{};
  {
    uint64_t dims[3] = {(uint64_t)D, (uint64_t)std::max<int64_t>(a->total_k, 1), (uint64_t)Hkv};
    uint64_t st[2] = {(uint64_t)Hkv * D, (uint64_t)D};
    const int hpc = Hkv % 4 == 0 ? 4 : (Hkv % 2 == 0 ? 2 : 1);
    p.heads_per_cta = hpc;
    uint32_t box[3] = {64, 32, (uint32_t)hpc};
    if ((rc = make_map(&p.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 3, a->k, dims, st, box, CU_TENSOR_MAP_SWIZZLE_128B)))
      return rc;
    if ((rc = make_map(&p.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 3, a->v, dims, st, box, CU_TENSOR_MAP_SWIZZLE_128B)))
      return rc;
  }
  p.q = a->q;
  p.out = a->out;
  p.cu_q = a->cu_seqlens_q;
  p.cu_k = a->cu_seqlens_k;
  p.num_seqs = a->num_seqs;
  p.total_q = a->total_q;
  p.total_k = a->total_k;
  p.hq = a->num_heads;
  p.hkv = Hkv;
  p.head_dim = D;
  p.scale_log2 = resolve_scale(a->scale, D) * kLog2e;
  p.status = static_cast<int*>(a->workspace);
  if ((rc = zero_status(a->workspace, s))) return rc;
  return launch_rc(launch_decode(p, s), "decode launch");
}

}  // extern "C"

// ------------------------------------------------------------------------ backward
namespace {

int make_bwd_maps(BwdParams* p, const void* q, const void* dout, const void* k, const void* v, float* dq_acc,
                  int64_t total_q, int64_t total_k, int H, int Hkv, int D) {
  int rc;
  if ((rc = map_thd(&p->tm_q, q, total_q, H, D, (int64_t)H * D, D, 64))) return rc;
  if ((rc = map_thd(&p->tm_do, dout, total_q, H, D, (int64_t)H * D, D, 64))) return rc;
  if ((rc = map_thd(&p->tm_k, k, total_k, Hkv, D, (int64_t)Hkv * D, D, 128))) return rc;
  if ((rc = map_thd(&p->tm_v, v, total_k, Hkv, D, (int64_t)Hkv * D, D, 128))) return rc;
  if ((rc = map_thd(&p->tm_k8, k, total_k, Hkv, D, (int64_t)Hkv * D, D, 8))) return rc;
  if ((rc = map_thd(&p->tm_v8, v, total_k, Hkv, D, (int64_t)Hkv * D, D, 8))) return rc;
  uint64_t dims[3] = {(uint64_t)D, (uint64_t)H, (uint64_t)std::max<int64_t>(total_q, 1)};
  uint64_t st[2] = {(uint64_t)D, (uint64_t)H * D};
  uint32_t box[3] = {(uint32_t)D / 4, 1, 16};  // one warp's head-dim slice x 16 q rows
  return make_map(&p->tm_dq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 3, dq_acc, dims, st, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

int64_t pad4(int64_t t) { return (t + 3) / 4 * 4; }

// [H, t_pad] pairs {lse * log2e, Delta} as a 2-D fp32 map, box of 66 pairs
int make_row_map(CUtensorMap* m, const float* rows, int64_t t_pad, int H) {
  uint64_t dims[2] = {(uint64_t)std::max<int64_t>(2 * t_pad, 8), (uint64_t)H};
  uint64_t st[1] = {(uint64_t)(2 * t_pad)};  // in elements
  uint32_t box[2] = {132, 1};
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 2, rows, dims, st, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

struct BwdLayout {
  Plan plan;
  size_t bytes = 0;
};

}  // namespace

extern "C" {

size_t cbv_zigzag_ring_bwd_workspace_size(const cbv_ring_args* a) {
  if (ring_common_checks(a)) return 0;
  Plan plan = plan_ring_bwd(a->cu_seqlens, a->num_docs, a->cp, (Layout)a->layout, a->window, a->num_kv_heads, 128);
  Carve c(nullptr);
  c.take(kStatusBytes);
  carve_plan(c, plan);
  c.take((size_t)a->num_heads * pad4(a->total) * sizeof(float));           // Delta
  c.take((size_t)a->num_heads * pad4(a->total) * sizeof(float));           // lse * log2e
  c.take(a->deterministic ? (size_t)fixed_tpad(a->total) * a->num_heads * a->head_dim * 8  // dq accumulator
                          : (size_t)a->total * a->num_heads * a->head_dim * 4);
  return c.off;
}

// Everything of the ring backward but the final dq conversion: dq stays in the accumulator
// carved from the workspace (fp32, or 64-bit fixed point when a->deterministic), returned
// through *dq_acc_out / *dq_fixed_out (the other one is set to null).
static int ring_bwd_core(const cbv_ring_args* a, cudaStream_t s, float** dq_acc_out,
                         unsigned long long** dq_fixed_out) {
  if (!a->dout || !a->out || !a->lse || !a->dk || !a->dv) return fail(CBV_ERR_BAD_ARG, "NULL tensor");
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->out) || !aligned16(a->dout) ||
      !aligned16(a->dk) || !aligned16(a->dv))
    return fail(CBV_ERR_MISALIGNED, "tensors must be 16-byte aligned");
  const int D = a->head_dim, H = a->num_heads, Hkv = a->num_kv_heads;
  const bool det = a->deterministic != 0;
  Plan plan = plan_ring_bwd(a->cu_seqlens, a->num_docs, a->cp, (Layout)a->layout, a->window, Hkv, 128);
  Carve c(a->workspace);
  int* status = static_cast<int*>(c.take(kStatusBytes));
  PlanDev pd = carve_plan(c, plan);
  const int64_t tp = pad4(a->total);
  float* rows = static_cast<float*>(c.take((size_t)H * tp * 2 * sizeof(float)));
  const size_t dq_bytes = det ? (size_t)fixed_tpad(a->total) * H * D * 8 : (size_t)a->total * H * D * 4;
  void* dq_buf = c.take(dq_bytes);
  if (!a->workspace || a->workspace_bytes < c.off) return fail(CBV_ERR_WORKSPACE_TOO_SMALL, "workspace needs %zu bytes", c.off);
  int rc;
  BwdParams p{};
  if ((rc = make_bwd_maps(&p, a->q, a->dout, a->k, a->v, static_cast<float*>(dq_buf), a->total, a->total, H, Hkv, D)))
    return rc;
  p.tasks = pd.tasks;
  p.segs = pd.segs;
  p.num_tasks = (int)plan.tasks.size();
  p.num_heads = H;
  p.num_kv_heads = Hkv;
  p.heads_per_kv = H / Hkv;
  p.scale = resolve_scale(a->scale, D);
  p.scale_log2 = p.scale * kLog2e;
  p.window = a->window > 0 ? a->window : 0;
  if ((rc = make_row_map(&p.tm_rows, rows, tp, H))) return rc;
  p.dk = a->dk;
  p.dv = a->dv;
  p.dkv_stride_t = (int64_t)Hkv * D;
  p.dkv_stride_h = D;
  p.dkv_accumulate = 0;
  p.dq_fixed = det ? static_cast<unsigned long long*>(dq_buf) : nullptr;
  p.dq_fixed_tpad = fixed_tpad(a->total);
  p.q_rows = p.kv_rows = a->total;
  p.prefetch_ahead = sm_count();
  p.status = status;
  if ((rc = upload_plan(pd, plan, s, status))) return rc;
  if ((rc = launch_rc(launch_bwd_preprocess(a->dout, a->out, a->lse, a->total, tp, H, D, rows,
                                            det ? nullptr : static_cast<float*>(dq_buf), det ? dq_buf : nullptr,
                                            det ? dq_bytes : 0, s),
                      "backward preprocess")))
    return rc;
  *dq_acc_out = det ? nullptr : static_cast<float*>(dq_buf);
  *dq_fixed_out = p.dq_fixed;
  return launch_rc(launch_bwd(p, D, grid_of(plan.tasks.size(), 1), s), "backward launch");
}

int cbv_zigzag_ring_bwd(const cbv_ring_args* a, void* stream) {
  NvtxRange nvtx_range("cbv_zigzag_ring_bwd");
  int rc = ring_common_checks(a);
  if (rc) return rc;
  if (a->total == 0) return CBV_OK;  // no rows: nothing to write
  if (!a->dq) return fail(CBV_ERR_BAD_ARG, "NULL tensor");
  if (!aligned16(a->dq)) return fail(CBV_ERR_MISALIGNED, "tensors must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* dq_acc = nullptr;
  unsigned long long* dq_fixed = nullptr;
  if ((rc = ring_bwd_core(a, s, &dq_acc, &dq_fixed))) return rc;
  const int64_t n = a->total * a->num_heads * a->head_dim;
  if (dq_fixed)
    return launch_rc(launch_fixed_to_bf16(dq_fixed, a->dq, a->total, a->num_heads, a->head_dim, s), "dq conversion");
  return launch_rc(launch_convert_bf16(dq_acc, a->dq, n, 1.f, s), "dq conversion");
}

static int block_bwd_checks(const cbv_block_bwd_args* a) {
  if (!a) return fail(CBV_ERR_BAD_ARG, "args is NULL");
  int rc = check_header(a->struct_size, sizeof(cbv_block_bwd_args), a->abi_version);
  if (rc) return rc;
  if ((rc = check_heads(a->num_heads, a->num_kv_heads, a->head_dim))) return rc;
  if ((rc = check_cu(a->cu_seqlens_q, a->num_docs, a->total_q, "cu_seqlens_q"))) return rc;
  if ((rc = check_cu(a->cu_seqlens_k, a->num_docs, a->total_k, "cu_seqlens_k"))) return rc;
  if (!a->dout || !a->q || !a->k || !a->v || !a->out || !a->lse || !a->dq_acc || !a->dk_acc || !a->dv_acc)
    return fail(CBV_ERR_BAD_ARG, "NULL tensor");
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->out) || !aligned16(a->dout) ||
      !aligned16(a->dq_acc) || !aligned16(a->dk_acc) || !aligned16(a->dv_acc))
    return fail(CBV_ERR_MISALIGNED, "tensors must be 16-byte aligned");
  return CBV_OK;
}

size_t cbv_block_bwd_workspace_size(const cbv_block_bwd_args* a) {
  if (block_bwd_checks(a)) return 0;
  Plan plan = plan_block_bwd(a->cu_seqlens_q, a->cu_seqlens_k, a->q_pos_base, a->k_pos_base, a->num_docs,
                             a->causal != 0, a->window, a->num_kv_heads, 128);
  Carve c(nullptr);
  c.take(kStatusBytes);
  carve_plan(c, plan);
  c.take((size_t)a->num_heads * pad4(a->total_q) * sizeof(float));
  c.take((size_t)a->num_heads * pad4(a->total_q) * sizeof(float));
  if (a->deterministic) c.take((size_t)fixed_tpad(a->total_q) * a->num_heads * a->head_dim * 8);  // fixed-point dq
  return c.off;
}

int cbv_attn_block_bwd(const cbv_block_bwd_args* a, void* stream) {
  NvtxRange nvtx_range("cbv_attn_block_bwd");
  int rc = block_bwd_checks(a);
  if (rc) return rc;
  if (a->total_q == 0 || a->total_k == 0) return CBV_OK;  // no (q, k) pair: the accumulators are unchanged
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = a->head_dim, H = a->num_heads, Hkv = a->num_kv_heads;
  Plan plan = plan_block_bwd(a->cu_seqlens_q, a->cu_seqlens_k, a->q_pos_base, a->k_pos_base, a->num_docs,
                             a->causal != 0, a->window, Hkv, 128);
  Carve c(a->workspace);
  int* status = static_cast<int*>(c.take(kStatusBytes));
  PlanDev pd = carve_plan(c, plan);
  const int64_t tp = pad4(a->total_q);
  float* rows = static_cast<float*>(c.take((size_t)H * tp * 2 * sizeof(float)));
  const size_t fix_bytes = a->deterministic ? (size_t)fixed_tpad(a->total_q) * H * D * 8 : 0;
  auto* dq_fixed = a->deterministic ? static_cast<unsigned long long*>(c.take(fix_bytes)) : nullptr;
  if (!a->workspace || a->workspace_bytes < c.off) return fail(CBV_ERR_WORKSPACE_TOO_SMALL, "workspace needs %zu bytes", c.off);
  BwdParams p{};
  if ((rc = make_bwd_maps(&p, a->q, a->dout, a->k, a->v, a->dq_acc, a->total_q, a->total_k, H, Hkv, D))) return rc;
  p.dq_fixed = dq_fixed;
  p.dq_fixed_tpad = fixed_tpad(a->total_q);
  p.q_rows = a->total_q;
  p.kv_rows = a->total_k;
  p.tasks = pd.tasks;
  p.segs = pd.segs;
  p.num_tasks = (int)plan.tasks.size();
  p.num_heads = H;
  p.num_kv_heads = Hkv;
  p.heads_per_kv = H / Hkv;
  p.scale = resolve_scale(a->scale, D);
  p.scale_log2 = p.scale * kLog2e;
  p.window = a->window > 0 ? a->window : 0;
  if ((rc = make_row_map(&p.tm_rows, rows, tp, H))) return rc;
  p.dk = a->dk_acc;
  p.dv = a->dv_acc;
  p.dkv_stride_t = (int64_t)Hkv * D;
  p.dkv_stride_h = D;
  p.dkv_accumulate = 1;
  p.prefetch_ahead = sm_count();
  p.status = status;
  if ((rc = upload_plan(pd, plan, s, status))) return rc;
  if ((rc = launch_rc(launch_bwd_preprocess(a->dout, a->out, a->lse, a->total_q, tp, H, D, rows, nullptr, dq_fixed,
                                            fix_bytes, s),
                      "backward preprocess")))
    return rc;
  if ((rc = launch_rc(launch_bwd(p, D, grid_of(plan.tasks.size(), 1), s), "backward launch"))) return rc;
  if (!dq_fixed) return CBV_OK;
  return launch_rc(launch_fixed_add_f32(dq_fixed, a->dq_acc, a->total_q, H, D, s), "dq accumulation");
}

}  // extern "C"

// ------------------------------------------------------------------------ EAGLE-3 cached ring
namespace {

// The ring arguments of block 0: the sequence keys and values are the first cache block.
cbv_ring_args cached_block0(const cbv_cached_ring_args* a) {
  cbv_ring_args r{};
  r.struct_size = sizeof(cbv_ring_args);
  r.abi_version = CBV_ABI_VERSION;
  r.q = a->q;
  r.k = a->cache_k ? a->cache_k[0] : nullptr;
  r.v = a->cache_v ? a->cache_v[0] : nullptr;
  r.total = a->total;
  r.num_heads = a->num_heads;
  r.num_kv_heads = a->num_kv_heads;
  r.head_dim = a->head_dim;
  r.num_docs = a->num_docs;
  r.cu_seqlens = a->cu_seqlens;
  r.max_seqlen = a->max_seqlen;
  r.cp = a->cp;
  r.layout = a->layout;
  r.scale = a->scale;
  r.causal = 1;
  r.window = a->window;
  r.schedule = CBV_SCHEDULE_FUSED;
  r.deterministic = a->deterministic;
  r.out = a->out;
  r.lse = a->lse;
  r.dout = a->dout;
  r.dq = a->dq;
  r.dk = a->dcache_k ? a->dcache_k[0] : nullptr;
  r.dv = a->dcache_v ? a->dcache_v[0] : nullptr;
  r.workspace = a->workspace;
  r.workspace_bytes = a->workspace_bytes;
  return r;
}

int cached_checks(const cbv_cached_ring_args* a) {
  if (!a) return fail(CBV_ERR_BAD_ARG, "args is NULL");
  int rc = check_header(a->struct_size, sizeof(cbv_cached_ring_args), a->abi_version);
  if (rc) return rc;
  if (a->num_blocks < 1 || a->num_blocks > cbv::kCacheMaxBlocks)
    return fail(CBV_ERR_BAD_ARG, "num_blocks must be in [1, %d]", cbv::kCacheMaxBlocks);
  cbv_ring_args r = cached_block0(a);
  return ring_common_checks(&r);
}

// The block addresses, checked: every block present and 16-byte aligned (gradients too when
// `grads`).
int cached_blocks(const cbv_cached_ring_args* a, bool grads, cbv::CacheBlocks* cb) {
  *cb = cbv::CacheBlocks{};
  if (!a->cache_k || !a->cache_v || (grads && (!a->dcache_k || !a->dcache_v)))
    return fail(CBV_ERR_BAD_ARG, "NULL cache block array");
  for (int i = 0; i < a->num_blocks; ++i) {
    cb->k[i] = a->cache_k[i];
    cb->v[i] = a->cache_v[i];
    if (grads) {
      cb->dk[i] = a->dcache_k[i];
      cb->dv[i] = a->dcache_v[i];
    }
    if (!cb->k[i] || !cb->v[i] || (grads && (!cb->dk[i] || !cb->dv[i])))
      return fail(CBV_ERR_BAD_ARG, "NULL cache block %d", i);
    if (!aligned16(cb->k[i]) || !aligned16(cb->v[i]) || (grads && (!aligned16(cb->dk[i]) || !aligned16(cb->dv[i]))))
      return fail(CBV_ERR_MISALIGNED, "cache block %d must be 16-byte aligned", i);
  }
  return CBV_OK;
}

size_t cached_fwd_bytes(const cbv_cached_ring_args* a, const RingFwdLayout& L) {
  size_t b = L.bytes;
  if (a->num_blocks > 1) b = (b + 255) / 256 * 256 + (size_t)a->total * a->num_heads * a->head_dim * sizeof(float);
  return b;
}

}  // namespace

extern "C" {

size_t cbv_cached_ring_fwd_workspace_size(const cbv_cached_ring_args* a) {
  if (cached_checks(a)) return 0;
  cbv_ring_args r = cached_block0(a);
  return cached_fwd_bytes(a, ring_fwd_layout(&r));
}

int cbv_cached_ring_fwd(const cbv_cached_ring_args* a, void* stream) {
  NvtxRange nvtx_range("cbv_cached_ring_fwd");
  int rc = cached_checks(a);
  if (rc) return rc;
  if (a->total == 0) return CBV_OK;
  cbv::CacheBlocks cb;
  if ((rc = cached_blocks(a, false, &cb))) return rc;
  cbv_ring_args r = cached_block0(a);
  if (a->num_blocks == 1) return cbv_zigzag_ring_fwd(&r, stream);  // the sequence alone
  if (!a->q || !a->out || !a->lse) return fail(CBV_ERR_BAD_ARG, "NULL tensor");
  if (!aligned16(a->q) || !aligned16(a->out)) return fail(CBV_ERR_MISALIGNED, "tensors must be 16-byte aligned");
  RingFwdLayout L = ring_fwd_layout(&r);
  const size_t need = cached_fwd_bytes(a, L);
  if (!a->workspace || a->workspace_bytes < need) return fail(CBV_ERR_WORKSPACE_TOO_SMALL, "workspace needs %zu bytes", need);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = a->head_dim, H = a->num_heads;
  Carve c(a->workspace);
  int* status = static_cast<int*>(c.take(kStatusBytes));
  PlanDev pd = carve_plan(c, L.fused);
  float* o32 = static_cast<float*>(c.take((size_t)a->total * H * D * sizeof(float)));
  FwdParams p = ring_fwd_params(&r, &rc);
  if (rc) return rc;
  p.status = status;
  if ((rc = upload_plan(pd, L.fused, s, status))) return rc;
  p.tasks = pd.tasks;
  p.segs = pd.segs;
  p.num_tasks = (int)L.fused.tasks.size();
  p.out = o32;  // block 0, normalised, fp32: the diagonals merge into it before rounding
  p.out_mode = kOutF32;
  if ((rc = launch_rc(launch_fwd_pingpong(p, D, false, grid_of(L.fused.tasks.size(), 1), s), "ring forward launch")))
    return rc;
  return launch_rc(cbv::launch_diag_merge(a->q, cb, a->num_blocks, a->total, H, a->num_kv_heads, D,
                                          resolve_scale(a->scale, D), o32, a->lse, a->out, s),
                   "diagonal merge");
}

size_t cbv_cached_ring_bwd_workspace_size(const cbv_cached_ring_args* a) {
  if (cached_checks(a)) return 0;
  cbv_ring_args r = cached_block0(a);
  return cbv_zigzag_ring_bwd_workspace_size(&r);
}

int cbv_cached_ring_bwd(const cbv_cached_ring_args* a, void* stream) {
  NvtxRange nvtx_range("cbv_cached_ring_bwd");
  int rc = cached_checks(a);
  if (rc) return rc;
  if (a->total == 0) return CBV_OK;
  cbv::CacheBlocks cb;
  if ((rc = cached_blocks(a, true, &cb))) return rc;
  cbv_ring_args r = cached_block0(a);
  if (a->num_blocks == 1) return cbv_zigzag_ring_bwd(&r, stream);
  if (!a->dq) return fail(CBV_ERR_BAD_ARG, "NULL tensor");
  if (!aligned16(a->dq)) return fail(CBV_ERR_MISALIGNED, "tensors must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* dq_acc = nullptr;
  unsigned long long* dq_fixed = nullptr;
  if ((rc = ring_bwd_core(&r, s, &dq_acc, &dq_fixed))) return rc;  // block 0 into dcache[0], dq kept unrounded
  const int D = a->head_dim;
  return launch_rc(cbv::launch_diag_grad(a->q, cb, a->num_blocks, a->total, a->num_heads, a->num_kv_heads, D,
                                         resolve_scale(a->scale, D), a->dout, a->out, a->lse, dq_acc, dq_fixed,
                                         a->dq, s),
                   "diagonal gradients");
}

}  // extern "C"

// ------------------------------------------------------------------------ one ring step on real ranks
namespace {

int ring_step_checks(const cbv_ring_step_args* a) {
  if (!a) return fail(CBV_ERR_BAD_ARG, "args is NULL");
  int rc = check_header(a->struct_size, sizeof(cbv_ring_step_args), a->abi_version);
  if (rc) return rc;
  if ((rc = check_heads(a->num_heads, a->num_kv_heads, a->head_dim))) return rc;
  if (a->cp < 1) return fail(CBV_ERR_BAD_ARG, "cp must be >= 1");
  if (a->rank < 0 || a->rank >= a->cp || a->step < 0 || a->step >= a->cp)
    return fail(CBV_ERR_BAD_ARG, "rank %d / step %d outside [0, %d)", a->rank, a->step, a->cp);
  if (a->layout != CBV_LAYOUT_ZIGZAG && a->layout != CBV_LAYOUT_CONTIGUOUS) return fail(CBV_ERR_BAD_ARG, "bad layout");
  if (a->n_local < 0) return fail(CBV_ERR_BAD_SHAPE, "n_local must be >= 0");
  if ((rc = check_cu(a->cu_seqlens, a->num_docs, a->n_local * a->cp, "cu_seqlens"))) return rc;
  if ((int64_t)a->cu_seqlens[a->num_docs] != a->n_local * a->cp)
    return fail(CBV_ERR_BAD_CU_SEQLENS, "cu_seqlens must end at n_local * cp (%lld)", (long long)(a->n_local * a->cp));
  std::string e = check_divisible(a->cu_seqlens, a->num_docs, a->cp, (Layout)a->layout);
  if (!e.empty()) return fail(CBV_ERR_NOT_DIVISIBLE_2CP, "%s", e.c_str());
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v)) return fail(CBV_ERR_MISALIGNED, "tensors must be 16-byte aligned");
  return CBV_OK;
}

Plan ring_step_fwd_plan(const cbv_ring_step_args* a) {
  return plan_ring_step_fwd(a->cu_seqlens, a->num_docs, a->cp, (Layout)a->layout, a->window, a->num_heads, a->rank,
                            a->step, kPairRows);
}

Plan ring_step_bwd_plan(const cbv_ring_step_args* a) {
  return plan_ring_step_bwd(a->cu_seqlens, a->num_docs, a->cp, (Layout)a->layout, a->window, a->num_kv_heads,
                            a->rank, a->step, 128);
}

}  // namespace

extern "C" {

size_t cbv_ring_step_fwd_workspace_size(const cbv_ring_step_args* a) {
  if (ring_step_checks(a)) return 0;
  Carve c(nullptr);
  c.take(kStatusBytes);
  carve_plan(c, ring_step_fwd_plan(a));
  return c.off;
}

int cbv_ring_step_fwd(const cbv_ring_step_args* a, void* stream) {
  NvtxRange nvtx_range("cbv_ring_step_fwd");
  int rc = ring_step_checks(a);
  if (rc) return rc;
  if (a->n_local == 0) return CBV_OK;
  if (!a->out_acc || !a->lse_acc) return fail(CBV_ERR_BAD_ARG, "NULL tensor");
  if (!aligned16(a->out_acc) || !aligned16(a->out)) return fail(CBV_ERR_MISALIGNED, "tensors must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = a->head_dim, H = a->num_heads, Hkv = a->num_kv_heads;
  Plan plan = ring_step_fwd_plan(a);
  Carve c(a->workspace);
  int* status = static_cast<int*>(c.take(kStatusBytes));
  PlanDev pd = carve_plan(c, plan);
  if (!a->workspace || a->workspace_bytes < c.off) return fail(CBV_ERR_WORKSPACE_TOO_SMALL, "workspace needs %zu bytes", c.off);
  FwdParams p{};
  if ((rc = map_thd(&p.tm_q, a->q, a->n_local, H, D, (int64_t)H * D, D, 128))) return rc;
  if ((rc = map_thd(&p.tm_k, a->k, a->n_local, Hkv, D, (int64_t)Hkv * D, D, 128))) return rc;
  if ((rc = map_thd(&p.tm_v, a->v, a->n_local, Hkv, D, (int64_t)Hkv * D, D, 128))) return rc;
  p.tasks = pd.tasks;
  p.segs = pd.segs;
  p.num_tasks = (int)plan.tasks.size();
  p.num_heads = H;
  p.heads_per_kv = H / Hkv;
  p.scale_log2 = resolve_scale(a->scale, D) * kLog2e;
  p.window = a->window > 0 ? a->window : 0;
  p.out = a->out_acc;
  p.out_stride_t = (int64_t)H * D;
  p.out_stride_h = D;
  p.lse = a->lse_acc;
  p.lse_stride_h = a->n_local;
  p.lse_stride_t = 1;
  p.out_mode = a->step == 0 ? kOutF32 : kOutMerge;  // every local row takes part in step 0's block
  p.block_size = 1;
  p.q_rows = p.kv_rows = a->n_local;
  p.status = status;
  if ((rc = upload_plan(pd, plan, s, status))) return rc;
  const int grid = grid_of(plan.tasks.size(), 1);
  if (grid < 0) return fail(CBV_ERR_BAD_SHAPE, "too many tiles");
  if ((rc = launch_rc(launch_fwd_pingpong(p, D, false, grid, s), "ring step forward launch"))) return rc;
  if (!a->out) return CBV_OK;
  return launch_rc(launch_convert_bf16(a->out_acc, a->out, a->n_local * H * D, 1.f, s), "output rounding");
}

size_t cbv_ring_step_bwd_workspace_size(const cbv_ring_step_args* a) {
  if (ring_step_checks(a)) return 0;
  Carve c(nullptr);
  c.take(kStatusBytes);
  carve_plan(c, ring_step_bwd_plan(a));
  c.take((size_t)a->num_heads * pad4(a->n_local) * 2 * sizeof(float));  // {lse * log2e, Delta}
  return c.off;
}

int cbv_ring_step_bwd(const cbv_ring_step_args* a, void* stream) {
  NvtxRange nvtx_range("cbv_ring_step_bwd");
  int rc = ring_step_checks(a);
  if (rc) return rc;
  if (a->n_local == 0) return CBV_OK;
  if (!a->dout || !a->out_merged || !a->lse_merged || !a->dq_acc || !a->dk_acc || !a->dv_acc)
    return fail(CBV_ERR_BAD_ARG, "NULL tensor");
  if (!aligned16(a->dout) || !aligned16(a->out_merged) || !aligned16(a->dq_acc) || !aligned16(a->dk_acc) ||
      !aligned16(a->dv_acc))
    return fail(CBV_ERR_MISALIGNED, "tensors must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = a->head_dim, H = a->num_heads, Hkv = a->num_kv_heads;
  Plan plan = ring_step_bwd_plan(a);
  Carve c(a->workspace);
  int* status = static_cast<int*>(c.take(kStatusBytes));
  PlanDev pd = carve_plan(c, plan);
  const int64_t tp = pad4(a->n_local);
  float* rows = static_cast<float*>(c.take((size_t)H * tp * 2 * sizeof(float)));
  if (!a->workspace || a->workspace_bytes < c.off) return fail(CBV_ERR_WORKSPACE_TOO_SMALL, "workspace needs %zu bytes", c.off);
  BwdParams p{};
  if ((rc = make_bwd_maps(&p, a->q, a->dout, a->k, a->v, a->dq_acc, a->n_local, a->n_local, H, Hkv, D))) return rc;
  p.tasks = pd.tasks;
  p.segs = pd.segs;
  p.num_tasks = (int)plan.tasks.size();
  p.num_heads = H;
  p.num_kv_heads = Hkv;
  p.heads_per_kv = H / Hkv;
  p.scale = resolve_scale(a->scale, D);
  p.scale_log2 = p.scale * kLog2e;
  p.window = a->window > 0 ? a->window : 0;
  if ((rc = make_row_map(&p.tm_rows, rows, tp, H))) return rc;
  p.dk = a->dk_acc;
  p.dv = a->dv_acc;
  p.dkv_stride_t = (int64_t)Hkv * D;
  p.dkv_stride_h = D;
  p.dkv_accumulate = 1;
  p.prefetch_ahead = sm_count();
  p.q_rows = p.kv_rows = a->n_local;
  p.status = status;
  if ((rc = upload_plan(pd, plan, s, status))) return rc;
  if ((rc = launch_rc(launch_bwd_preprocess(a->dout, a->out_merged, a->lse_merged, a->n_local, tp, H, D, rows, nullptr,
                                            nullptr, 0, s),
                      "backward preprocess")))
    return rc;
  return launch_rc(launch_bwd(p, D, grid_of(plan.tasks.size(), 1), s), "ring step backward launch");
}

// ------------------------------------------------------------------------ cache diagonals alone
static int diag_checks(const cbv_diag_args* a, cbv::CacheBlocks* cb, bool grads) {
  if (!a) return fail(CBV_ERR_BAD_ARG, "args is NULL");
  int rc = check_header(a->struct_size, sizeof(cbv_diag_args), a->abi_version);
  if (rc) return rc;
  if ((rc = check_heads(a->num_heads, a->num_kv_heads, a->head_dim))) return rc;
  if (a->num_blocks < 1 || a->num_blocks > cbv::kCacheMaxBlocks)
    return fail(CBV_ERR_BAD_ARG, "num_blocks must be in [1, %d]", cbv::kCacheMaxBlocks);
  if (a->total < 0) return fail(CBV_ERR_BAD_SHAPE, "total must be >= 0");
  *cb = cbv::CacheBlocks{};
  if (a->num_blocks > 1 && (!a->cache_k || !a->cache_v || (grads && (!a->dcache_k || !a->dcache_v))))
    return fail(CBV_ERR_BAD_ARG, "NULL cache block array");
  for (int i = 1; i < a->num_blocks; ++i) {
    cb->k[i] = a->cache_k[i];
    cb->v[i] = a->cache_v[i];
    if (grads) {
      cb->dk[i] = a->dcache_k[i];
      cb->dv[i] = a->dcache_v[i];
    }
    if (!cb->k[i] || !cb->v[i] || (grads && (!cb->dk[i] || !cb->dv[i]))) return fail(CBV_ERR_BAD_ARG, "NULL cache block %d", i);
    if (!aligned16(cb->k[i]) || !aligned16(cb->v[i]) || (grads && (!aligned16(cb->dk[i]) || !aligned16(cb->dv[i]))))
      return fail(CBV_ERR_MISALIGNED, "cache block %d must be 16-byte aligned", i);
  }
  return CBV_OK;
}

int cbv_cached_diag_merge(const cbv_diag_args* a, void* stream) {
  NvtxRange nvtx_range("cbv_cached_diag_merge");
  cbv::CacheBlocks cb;
  int rc = diag_checks(a, &cb, false);
  if (rc) return rc;
  if (a->total == 0) return CBV_OK;
  if (!a->q || !a->out0 || !a->lse || !a->out) return fail(CBV_ERR_BAD_ARG, "NULL tensor");
  if (!aligned16(a->q) || !aligned16(a->out0) || !aligned16(a->out)) return fail(CBV_ERR_MISALIGNED, "tensors must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = a->head_dim, H = a->num_heads;
  if (a->num_blocks == 1)
    return launch_rc(launch_convert_bf16(a->out0, a->out, a->total * H * D, 1.f, s), "output rounding");
  return launch_rc(cbv::launch_diag_merge(a->q, cb, a->num_blocks, a->total, H, a->num_kv_heads, D,
                                          resolve_scale(a->scale, D), a->out0, a->lse, a->out, s),
                   "diagonal merge");
}

int cbv_cached_diag_grad(const cbv_diag_args* a, void* stream) {
  NvtxRange nvtx_range("cbv_cached_diag_grad");
  cbv::CacheBlocks cb;
  int rc = diag_checks(a, &cb, true);
  if (rc) return rc;
  if (a->total == 0) return CBV_OK;
  if (!a->dq0 || !a->dq || (a->num_blocks > 1 && (!a->q || !a->dout || !a->out_merged || !a->lse_merged)))
    return fail(CBV_ERR_BAD_ARG, "NULL tensor");
  if (!aligned16(a->dq0) || !aligned16(a->dq) || !aligned16(a->q) || !aligned16(a->dout) || !aligned16(a->out_merged))
    return fail(CBV_ERR_MISALIGNED, "tensors must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = a->head_dim, H = a->num_heads;
  if (a->num_blocks == 1) return launch_rc(launch_convert_bf16(a->dq0, a->dq, a->total * H * D, 1.f, s), "dq rounding");
  return launch_rc(cbv::launch_diag_grad(a->q, cb, a->num_blocks, a->total, H, a->num_kv_heads, D,
                                         resolve_scale(a->scale, D), a->dout, a->out_merged, a->lse_merged, a->dq0,
                                         nullptr, a->dq, s),
                   "diagonal gradients");
}

// ------------------------------------------------------------------------ layout helpers
int cbv_convert_f32_bf16(const float* src, void* dst, int64_t n, float mul, void* stream) {
  if (n < 0 || n % 4) return fail(CBV_ERR_BAD_SHAPE, "n must be a non-negative multiple of 4");
  if (n == 0) return CBV_OK;
  if (!src || !dst) return fail(CBV_ERR_BAD_ARG, "NULL tensor");
  if (!aligned16(src) || !aligned16(dst)) return fail(CBV_ERR_MISALIGNED, "tensors must be 16-byte aligned");
  return launch_rc(launch_convert_bf16(src, dst, n, mul, static_cast<cudaStream_t>(stream)), "conversion");
}

int cbv_swap_leading_axes(const void* src, void* dst, int64_t a, int64_t b, int64_t row_bytes, void* stream) {
  if (a < 0 || b < 0 || row_bytes < 0 || row_bytes % 4) return fail(CBV_ERR_BAD_SHAPE, "bad sizes");
  if (a * b * row_bytes == 0) return CBV_OK;
  if (!src || !dst) return fail(CBV_ERR_BAD_ARG, "NULL tensor");
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 3) return fail(CBV_ERR_MISALIGNED, "4-byte alignment");
  const char *s0 = static_cast<const char*>(src), *d0 = static_cast<const char*>(dst);
  const int64_t n = a * b * row_bytes;
  if (s0 < d0 + n && d0 < s0 + n) return fail(CBV_ERR_BAD_ARG, "src and dst overlap");
  return launch_rc(launch_swap01(src, dst, a, b, row_bytes, static_cast<cudaStream_t>(stream)), "axis swap");
}

}  // extern "C"
