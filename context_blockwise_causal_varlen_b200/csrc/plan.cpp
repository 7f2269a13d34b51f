// Host planner (see plan.h).
#include "plan.h"

#include <algorithm>
#include <cstdio>
#include <map>
#include <tuple>

namespace cbv {

namespace {

int64_t sum_capped(int64_t a, int64_t b, int64_t window) {
  // sum_{i=a}^{b-1} min(i + 1, window), window <= 0 meaning no cap
  if (b <= a) return 0;
  if (window <= 0) return (b * (b + 1) - a * (a + 1)) / 2;
  int64_t s = 0;
  int64_t lo = a, hi = std::min(b, window);  // i + 1 <= window  <=>  i < window
  if (hi > lo) s += (hi * (hi + 1) - lo * (lo + 1)) / 2;
  int64_t rest = b - std::max(a, window);
  if (rest > 0) s += rest * window;
  return s;
}

// sum over q in [q0, q1) of clamp(q - a, 0, n): a ramp that starts after q = a and saturates at n
int64_t ramp_sum(int64_t q0, int64_t q1, int64_t a, int64_t n) {
  int64_t s = 0;
  const int64_t lo = std::max(q0, a + 1), hi = std::min(q1, a + n);
  if (hi > lo) s += (hi - lo) * ((lo - a) + (hi - 1 - a)) / 2;
  const int64_t lo2 = std::max(q0, a + n);
  if (q1 > lo2) s += (q1 - lo2) * n;
  return s;
}

// visible (q, k) pairs between q positions [qp, qp+nq) and k positions [kp, kp+nk): with the
// causal or window test, the pairs with 0 <= q - k (and q - k < window), counted as the pairs with
// q - k >= 0 minus those with q - k >= window; each count is a ramp sum over q
int64_t visible_pairs(int64_t qp, int64_t nq, int64_t kp, int64_t nk, bool causal, int64_t window) {
  if (nq <= 0 || nk <= 0) return 0;
  if (!causal && window <= 0) return nq * nk;
  const int64_t ahead = ramp_sum(qp, qp + nq, kp - 1, nk);
  if (window <= 0) return ahead;
  return ahead - ramp_sum(qp, qp + nq, kp - 1 + window, nk);
}

int32_t weight(int64_t pairs) { return (int32_t)std::min<int64_t>(pairs / 256 + 1, INT32_MAX); }

// Replace segs[first..] by their union as runs of adjacent rows, in position order.
// A run is causal if any of its parts is (the causal test is a no-op on parts that
// lie wholly before the tile, so applying it to the whole run changes nothing).
void coalesce_tail(std::vector<Seg>& segs, size_t first) {
  std::vector<Seg> part(segs.begin() + first, segs.end());
  std::sort(part.begin(), part.end(), [](const Seg& a, const Seg& b) { return a.row0 < b.row0; });
  segs.resize(first);
  for (const Seg& s : part) {
    if (segs.size() > first) {
      Seg& t = segs.back();
      if (t.row0 + t.rows == s.row0 && t.pos0 + t.rows == s.pos0) {
        t.rows += s.rows;
        t.flags |= (s.flags & kSegCausal);
        continue;
      }
    }
    segs.push_back(s);
  }
  if (segs.size() > first) segs[first].flags |= kSegBlockStart;
}

// Expands every tile (whose `head` field holds its group, e.g. its document) into one
// task per head, ordered so that tasks sharing operands run side by side: groups by
// descending total work, inside a group head by head (heads of one GQA group are
// adjacent), inside a head tiles by descending work.  Consecutive CTAs then reuse the
// same k/v (forward) or q/dO and dq rows (backward) from L2, and the largest pieces
// start first.  Fills plan.tasks and its compact form (plan.tiles, plan.groups).
void expand_heads(Plan& plan, int32_t heads) {
  std::map<int32_t, std::vector<TileTask>> groups;
  std::map<int32_t, int64_t> total;
  for (const TileTask& t : plan.tasks) {
    groups[t.head].push_back(t);
    total[t.head] += t.work;
  }
  std::vector<int32_t> order;
  for (auto& kv : groups) order.push_back(kv.first);
  std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) { return total[a] > total[b]; });
  std::vector<TileTask> out;
  out.reserve(plan.tasks.size() * (size_t)heads);
  plan.tiles.clear();
  plan.groups.clear();
  for (int32_t g : order) {
    auto& v = groups[g];
    std::stable_sort(v.begin(), v.end(), [](const TileTask& a, const TileTask& b) { return a.work > b.work; });
    plan.groups.push_back({(int32_t)out.size(), (int32_t)plan.tiles.size(), (int32_t)v.size(), 0});
    for (TileTask t : v) {
      t.head = 0;
      plan.tiles.push_back(t);
    }
    for (int32_t h = 0; h < heads; ++h)
      for (TileTask t : v) {
        t.head = h;
        out.push_back(t);
      }
  }
  plan.tasks.swap(out);
}

}  // namespace

std::string check_cu_seqlens(const int32_t* cu, int32_t num_docs) {
  if (num_docs < 0) return "num_docs must be >= 0";
  if (cu == nullptr) return "cu_seqlens is NULL";
  if (cu[0] != 0) return "cu_seqlens[0] must be 0";
  for (int32_t d = 0; d < num_docs; ++d)
    if (cu[d + 1] < cu[d]) return "cu_seqlens must be non-decreasing";
  return "";
}

std::string check_divisible(const int32_t* cu, int32_t num_docs, int32_t cp, Layout layout) {
  if (cp < 1) return "cp must be >= 1";
  const int32_t n = layout == kZigZag ? 2 * cp : cp;
  for (int32_t d = 0; d < num_docs; ++d)
    if ((cu[d + 1] - cu[d]) % n) {
      char buf[160];
      snprintf(buf, sizeof buf, "document %d has length %d, not divisible by %d", d, cu[d + 1] - cu[d], n);
      return buf;
    }
  return "";
}

void local_cu_seqlens(const int32_t* cu, int32_t num_docs, int32_t cp, int32_t* out) {
  for (int32_t d = 0; d <= num_docs; ++d) out[d] = cu[d] / cp;
}

void half_cu_seqlens(const int32_t* cu, int32_t num_docs, int32_t cp, int32_t* out) {
  for (int32_t d = 0; d <= num_docs; ++d) out[d] = cu[d] / (2 * cp);
}

int64_t get_half_index(const int32_t* cu_local, int32_t num_docs, bool front, int32_t* out) {
  int64_t n = 0;
  for (int32_t d = 0; d < num_docs; ++d) {
    const int32_t a = cu_local[d], b = cu_local[d + 1], mid = a + (b - a) / 2;
    const int32_t lo = front ? a : mid, hi = front ? mid : b;
    for (int32_t i = lo; i < hi; ++i) {
      if (out) out[n] = i;
      ++n;
    }
  }
  return n;
}

int64_t rank_tokens(const int32_t* cu, int32_t num_docs, int32_t cp, int32_t rank, Layout layout, int32_t* out) {
  int64_t n = 0;
  auto emit = [&](int32_t a, int32_t b) {
    for (int32_t i = a; i < b; ++i) {
      if (out) out[n] = i;
      ++n;
    }
  };
  for (int32_t d = 0; d < num_docs; ++d) {
    const int32_t g = cu[d], L = cu[d + 1] - cu[d];
    if (layout == kZigZag) {
      const int32_t c = L / (2 * cp);
      emit(g + rank * c, g + (rank + 1) * c);
      emit(g + (2 * cp - 1 - rank) * c, g + (2 * cp - rank) * c);
    } else {
      const int32_t c = L / cp;
      emit(g + rank * c, g + (rank + 1) * c);
    }
  }
  return n;
}

void rank_pair_counts(const int32_t* cu, int32_t num_docs, int32_t cp, Layout layout, int32_t window, int64_t* out) {
  for (int32_t r = 0; r < cp; ++r) {
    int64_t s = 0;
    for (int32_t d = 0; d < num_docs; ++d) {
      const int64_t L = cu[d + 1] - cu[d];
      if (layout == kZigZag) {
        const int64_t c = L / (2 * cp);
        s += sum_capped(r * c, (r + 1) * c, window);
        s += sum_capped((2 * cp - 1 - r) * c, (2 * cp - r) * c, window);
      } else {
        const int64_t c = L / cp;
        s += sum_capped(r * c, (r + 1) * c, window);
      }
    }
    out[r] = s;
  }
}

void ring_step(int32_t rank, int32_t step, int32_t cp, Layout layout, int32_t* src, int32_t* kind) {
  *src = ((rank - step) % cp + cp) % cp;
  if (step == 0) {
    *kind = kDiag;
  } else if (layout == kZigZag) {
    *kind = *src < rank ? kFrontK : kBackQ;
  } else {
    *kind = step <= rank ? kFull : kSkip;
  }
}

void ring_blocks(const int32_t* cu, int32_t num_docs, int32_t cp, Layout layout, std::vector<RingBlock>* blocks,
                 std::vector<RowRun>* runs) {
  blocks->clear();
  runs->clear();
  const int32_t nchunk = layout == kZigZag ? 2 * cp : cp;
  // the run of chunk x of document d, which is local chunk `part` (0 front, 1 back) of its rank
  auto chunk_run = [&](int32_t d, int32_t x, int32_t part) {
    const int32_t c = (cu[d + 1] - cu[d]) / nchunk;
    const int32_t row0 = cu[d] + x * c;
    runs->push_back({d, row0, c, row0, cu[d] / cp + part * c});
  };
  for (int32_t r = 0; r < cp; ++r) {
    for (int32_t s = 0; s < cp; ++s) {
      int32_t src, kind;
      ring_step(r, s, cp, layout, &src, &kind);
      if (kind == kSkip) continue;
      RingBlock b{};
      b.rank = r;
      b.step = s;
      b.src = src;
      b.kind = kind;
      b.causal = kind == kDiag;
      b.q_half = kind == kBackQ ? 2 : 0;
      b.k_half = kind == kFrontK ? 1 : 0;
      // q runs: rank r's local rows (or back halves); k runs: src's local rows (or front halves)
      b.q_run0 = (int32_t)runs->size();
      for (int32_t d = 0; d < num_docs; ++d) {
        if (cu[d + 1] == cu[d]) continue;
        if (layout == kContiguous) {
          chunk_run(d, r, 0);
          continue;
        }
        if (b.q_half != 2) chunk_run(d, r, 0);
        chunk_run(d, 2 * cp - 1 - r, 1);
      }
      b.q_nruns = (int32_t)runs->size() - b.q_run0;
      b.k_run0 = (int32_t)runs->size();
      for (int32_t d = 0; d < num_docs; ++d) {
        if (cu[d + 1] == cu[d]) continue;
        if (layout == kContiguous) {
          chunk_run(d, src, 0);
          continue;
        }
        chunk_run(d, src, 0);
        if (b.k_half != 1) chunk_run(d, 2 * cp - 1 - src, 1);
      }
      b.k_nruns = (int32_t)runs->size() - b.k_run0;
      blocks->push_back(b);
    }
  }
}

std::vector<ChunkPair> ring_chunk_pairs(const int32_t* cu, int32_t num_docs, int32_t cp, Layout layout,
                                        int32_t window, int32_t only_step) {
  std::vector<ChunkPair> out;
  for (int32_t r = 0; r < cp; ++r) {
    for (int32_t s = 0; s < cp; ++s) {
      if (only_step >= 0 && s != only_step) continue;
      int32_t src, kind;
      ring_step(r, s, cp, layout, &src, &kind);
      if (kind == kSkip) continue;
      for (int32_t d = 0; d < num_docs; ++d) {
        const int32_t L = cu[d + 1] - cu[d];
        const int32_t nchunk = layout == kZigZag ? 2 * cp : cp;
        const int32_t c = L / nchunk;
        if (c == 0) continue;
        std::vector<std::tuple<int32_t, int32_t, int32_t>> p;  // (q chunk, k chunk, causal)
        if (layout == kZigZag) {
          const int32_t f = r, b = 2 * cp - 1 - r, fs = src, bs = 2 * cp - 1 - src;
          if (kind == kDiag) p = {{f, f, 1}, {b, f, 0}, {b, b, 1}};
          else if (kind == kFrontK) p = {{f, fs, 0}, {b, fs, 0}};
          else p = {{b, fs, 0}, {b, bs, 0}};
        } else {
          if (kind == kDiag) p = {{r, r, 1}};
          else p = {{r, src, 0}};
        }
        for (auto& [x, y, causal] : p) {
          // with a sliding window, drop chunk pairs that no query of x can see
          if (window > 0 && x > y && (int64_t)(x - y - 1) * c + 1 >= window) continue;
          out.push_back({d, r, s, x, y, causal});
        }
      }
    }
  }
  return out;
}

Plan plan_ring_fwd(const int32_t* cu, int32_t num_docs, int32_t cp, Layout layout, int32_t window, int32_t heads,
                   int32_t only_step, int32_t tile_m, bool coalesce) {
  Plan plan;
  const int32_t nchunk = layout == kZigZag ? 2 * cp : cp;
  std::vector<ChunkPair> pairs = ring_chunk_pairs(cu, num_docs, cp, layout, window, only_step);
  // group by (doc, q chunk), keeping ring order
  std::map<std::pair<int32_t, int32_t>, std::vector<ChunkPair>> groups;
  std::vector<std::pair<int32_t, int32_t>> order;
  for (auto& p : pairs) {
    auto key = std::make_pair(p.doc, p.q_chunk);
    if (!groups.count(key)) order.push_back(key);
    groups[key].push_back(p);
  }
  for (auto& key : order) {
    const auto& g = groups[key];
    const int32_t d = key.first, x = key.second;
    const int32_t c = (cu[d + 1] - cu[d]) / nchunk;
    const int32_t seg0 = (int32_t)plan.segs.size();
    int32_t last_step = -1;
    for (auto& p : g) {
      Seg s;
      s.row0 = cu[d] + p.k_chunk * c;
      s.rows = c;
      s.pos0 = s.row0;
      s.flags = (p.causal ? kSegCausal : 0) | (p.step != last_step ? kSegBlockStart : 0);
      last_step = p.step;
      plan.segs.push_back(s);
    }
    if (coalesce) coalesce_tail(plan.segs, seg0);
    const int32_t nseg = (int32_t)plan.segs.size() - seg0;
    for (int32_t t0 = 0; t0 < c; t0 += tile_m) {
      TileTask t{};
      t.row0 = cu[d] + x * c + t0;
      t.rows = std::min(tile_m, c - t0);
      t.pos0 = t.row0;
      t.seg0 = seg0;
      t.nseg = nseg;
      t.aux = -1;
      t.head = d;
      int64_t w = 0;
      for (int32_t i = 0; i < nseg; ++i) {
        const Seg& s = plan.segs[seg0 + i];
        w += visible_pairs(t.pos0, t.rows, s.pos0, s.rows, s.flags & kSegCausal, window);
      }
      t.work = weight(w);
      plan.tasks.push_back(t);
    }
  }
  expand_heads(plan, heads);
  return plan;
}

Plan plan_ring_bwd(const int32_t* cu, int32_t num_docs, int32_t cp, Layout layout, int32_t window, int32_t kv_heads,
                   int32_t tile_n) {
  Plan plan;
  const int32_t nchunk = layout == kZigZag ? 2 * cp : cp;
  std::vector<ChunkPair> pairs = ring_chunk_pairs(cu, num_docs, cp, layout, window, -1);
  std::map<std::pair<int32_t, int32_t>, std::vector<ChunkPair>> groups;
  std::vector<std::pair<int32_t, int32_t>> order;
  for (auto& p : pairs) {
    auto key = std::make_pair(p.doc, p.k_chunk);
    if (!groups.count(key)) order.push_back(key);
    groups[key].push_back(p);
  }
  for (auto& key : order) {
    const auto& g = groups[key];
    const int32_t d = key.first, y = key.second;
    const int32_t c = (cu[d + 1] - cu[d]) / nchunk;
    const int32_t seg0 = (int32_t)plan.segs.size();
    for (auto& p : g) {
      Seg s;
      s.row0 = cu[d] + p.q_chunk * c;
      s.rows = c;
      s.pos0 = s.row0;
      s.flags = (p.causal ? kSegCausal : 0) | kSegBlockStart;
      plan.segs.push_back(s);
    }
    coalesce_tail(plan.segs, seg0);
    const int32_t nseg = (int32_t)plan.segs.size() - seg0;
    // Zig-zag without a window: a rank's two chunks of a document, f < cp and b = 2cp-1-f, end in
    // equally ragged key tiles.  When the two tails fit in one tile they share it: the keys of
    // chunk b are seen only by q rows of chunks >= b, all of them among chunk f's segments, so
    // the tile walks chunk f's segments and masks by position.  Chunk b's tail gets no task.
    const int32_t tail = c % tile_n;
    const bool pair_tails = layout == kZigZag && window <= 0 && tail > 0 && tail <= tile_n / 2;
    for (int32_t t0 = 0; t0 < c; t0 += tile_n) {
      const bool is_tail = t0 + tile_n > c;
      if (pair_tails && is_tail && y >= cp) continue;  // rides in chunk f's tail tile
      TileTask t{};
      t.row0 = cu[d] + y * c + t0;
      t.rows = std::min(tile_n, c - t0);
      t.pos0 = t.row0;
      t.seg0 = seg0;
      t.nseg = nseg;
      t.aux = -1;
      t.head = d;
      if (pair_tails && is_tail) {
        t.row1 = cu[d] + (nchunk - 1 - y) * c + t0;
        t.pos1 = t.row1;
        t.rows1 = tail;
        t.split1 = (tail + 7) / 8 * 8;
      }
      int64_t w = 0;
      for (int32_t i = 0; i < nseg; ++i) {
        const Seg& s = plan.segs[seg0 + i];
        w += visible_pairs(s.pos0, s.rows, t.pos0, t.rows, s.flags & kSegCausal, window);
        if (t.split1) w += visible_pairs(s.pos0, s.rows, t.pos1, t.rows1, s.flags & kSegCausal, window);
      }
      t.work = weight(w);
      plan.tasks.push_back(t);
    }
  }
  expand_heads(plan, kv_heads);
  return plan;
}

namespace {

// First row of global chunk x of document d in the local sequence of the rank that owns it (its
// front chunk first, then its back chunk).
int32_t chunk_local0(const int32_t* cu, int32_t d, int32_t x, int32_t cp, Layout layout) {
  const int32_t nchunk = layout == kZigZag ? 2 * cp : cp;
  const int32_t c = (cu[d + 1] - cu[d]) / nchunk;
  return cu[d] / cp + ((layout == kZigZag && x >= cp) ? c : 0);
}

// The chunk pairs of `rank` at `step`, grouped by (document, chunk of side `key`), in order.
std::vector<std::vector<ChunkPair>> step_groups(const int32_t* cu, int32_t num_docs, int32_t cp, Layout layout,
                                                int32_t window, int32_t rank, int32_t step, bool by_k) {
  std::map<std::pair<int32_t, int32_t>, size_t> at;
  std::vector<std::vector<ChunkPair>> out;
  for (const ChunkPair& p : ring_chunk_pairs(cu, num_docs, cp, layout, window, step)) {
    if (p.rank != rank) continue;
    const auto key = std::make_pair(p.doc, by_k ? p.k_chunk : p.q_chunk);
    auto it = at.find(key);
    if (it == at.end()) {
      at[key] = out.size();
      out.push_back({p});
    } else {
      out[it->second].push_back(p);
    }
  }
  return out;
}

}  // namespace

Plan plan_ring_step_fwd(const int32_t* cu, int32_t num_docs, int32_t cp, Layout layout, int32_t window,
                        int32_t heads, int32_t rank, int32_t step, int32_t tile_m) {
  Plan plan;
  const int32_t nchunk = layout == kZigZag ? 2 * cp : cp;
  for (const auto& g : step_groups(cu, num_docs, cp, layout, window, rank, step, false)) {
    const int32_t d = g[0].doc, x = g[0].q_chunk;
    const int32_t c = (cu[d + 1] - cu[d]) / nchunk;
    const int32_t seg0 = (int32_t)plan.segs.size();
    for (const ChunkPair& p : g) {
      Seg s;
      s.row0 = chunk_local0(cu, d, p.k_chunk, cp, layout);
      s.rows = c;
      s.pos0 = cu[d] + p.k_chunk * c;
      s.flags = (p.causal ? kSegCausal : 0) | (p.k_chunk == g[0].k_chunk ? kSegBlockStart : 0);
      plan.segs.push_back(s);
    }
    coalesce_tail(plan.segs, seg0);
    const int32_t nseg = (int32_t)plan.segs.size() - seg0;
    for (int32_t t0 = 0; t0 < c; t0 += tile_m) {
      TileTask t{};
      t.row0 = chunk_local0(cu, d, x, cp, layout) + t0;
      t.rows = std::min(tile_m, c - t0);
      t.pos0 = cu[d] + x * c + t0;
      t.seg0 = seg0;
      t.nseg = nseg;
      t.aux = -1;
      t.head = d;
      int64_t w = 0;
      for (int32_t i = 0; i < nseg; ++i) {
        const Seg& s = plan.segs[seg0 + i];
        w += visible_pairs(t.pos0, t.rows, s.pos0, s.rows, s.flags & kSegCausal, window);
      }
      t.work = weight(w);
      plan.tasks.push_back(t);
    }
  }
  expand_heads(plan, heads);
  return plan;
}

Plan plan_ring_step_bwd(const int32_t* cu, int32_t num_docs, int32_t cp, Layout layout, int32_t window,
                        int32_t kv_heads, int32_t rank, int32_t step, int32_t tile_n) {
  Plan plan;
  const int32_t nchunk = layout == kZigZag ? 2 * cp : cp;
  for (const auto& g : step_groups(cu, num_docs, cp, layout, window, rank, step, true)) {
    const int32_t d = g[0].doc, y = g[0].k_chunk;
    const int32_t c = (cu[d + 1] - cu[d]) / nchunk;
    const int32_t seg0 = (int32_t)plan.segs.size();
    for (const ChunkPair& p : g) {
      Seg s;
      s.row0 = chunk_local0(cu, d, p.q_chunk, cp, layout);
      s.rows = c;
      s.pos0 = cu[d] + p.q_chunk * c;
      s.flags = (p.causal ? kSegCausal : 0) | kSegBlockStart;
      plan.segs.push_back(s);
    }
    coalesce_tail(plan.segs, seg0);
    const int32_t nseg = (int32_t)plan.segs.size() - seg0;
    for (int32_t t0 = 0; t0 < c; t0 += tile_n) {
      TileTask t{};
      t.row0 = chunk_local0(cu, d, y, cp, layout) + t0;
      t.rows = std::min(tile_n, c - t0);
      t.pos0 = cu[d] + y * c + t0;
      t.seg0 = seg0;
      t.nseg = nseg;
      t.aux = -1;
      t.head = d;
      int64_t w = 0;
      for (int32_t i = 0; i < nseg; ++i) {
        const Seg& s = plan.segs[seg0 + i];
        w += visible_pairs(s.pos0, s.rows, t.pos0, t.rows, s.flags & kSegCausal, window);
      }
      t.work = weight(w);
      plan.tasks.push_back(t);
    }
  }
  expand_heads(plan, kv_heads);
  return plan;
}

Plan plan_block_fwd(const int32_t* cu_q, const int32_t* cu_k, const int32_t* qbase, const int32_t* kbase,
                    int32_t num_docs, bool causal, int32_t window, int32_t heads, int32_t tile_m) {
  Plan plan;
  for (int32_t d = 0; d < num_docs; ++d) {
    const int32_t lq = cu_q[d + 1] - cu_q[d], lk = cu_k[d + 1] - cu_k[d];
    if (lq == 0) continue;
    const int32_t qb = qbase ? qbase[d] : lk - lq;
    const int32_t kb = kbase ? kbase[d] : 0;
    const int32_t seg0 = (int32_t)plan.segs.size();
    if (lk > 0) plan.segs.push_back(Seg{cu_k[d], lk, kb, (causal ? kSegCausal : 0) | kSegBlockStart});
    const int32_t nseg = (int32_t)plan.segs.size() - seg0;
    for (int32_t t0 = 0; t0 < lq; t0 += tile_m) {
      TileTask t{};
      t.row0 = cu_q[d] + t0;
      t.rows = std::min(tile_m, lq - t0);
      t.pos0 = qb + t0;
      t.seg0 = seg0;
      t.nseg = nseg;
      t.aux = -1;
      t.head = d;
      t.work = nseg ? weight(visible_pairs(t.pos0, t.rows, kb, lk, causal, window)) : 0;
      plan.tasks.push_back(t);
    }
  }
  expand_heads(plan, heads);
  return plan;
}

Plan plan_block_bwd(const int32_t* cu_q, const int32_t* cu_k, const int32_t* qbase, const int32_t* kbase,
                    int32_t num_docs, bool causal, int32_t window, int32_t kv_heads, int32_t tile_n) {
  Plan plan;
  for (int32_t d = 0; d < num_docs; ++d) {
    const int32_t lq = cu_q[d + 1] - cu_q[d], lk = cu_k[d + 1] - cu_k[d];
    if (lk == 0) continue;
    const int32_t qb = qbase ? qbase[d] : lk - lq;
    const int32_t kb = kbase ? kbase[d] : 0;
    const int32_t seg0 = (int32_t)plan.segs.size();
    if (lq > 0) plan.segs.push_back(Seg{cu_q[d], lq, qb, (causal ? kSegCausal : 0) | kSegBlockStart});
    const int32_t nseg = (int32_t)plan.segs.size() - seg0;
    for (int32_t t0 = 0; t0 < lk; t0 += tile_n) {
      TileTask t{};
      t.row0 = cu_k[d] + t0;
      t.rows = std::min(tile_n, lk - t0);
      t.pos0 = kb + t0;
      t.seg0 = seg0;
      t.nseg = nseg;
      t.aux = -1;
      t.head = d;
      t.work = nseg ? weight(visible_pairs(qb, lq, t.pos0, t.rows, causal, window)) : 0;
      plan.tasks.push_back(t);
    }
  }
  expand_heads(plan, kv_heads);
  return plan;
}

Plan plan_kvp(int32_t q_len, int32_t heads, int32_t shards, int32_t n_local, int32_t seg_size, KvMode mode,
              int32_t block_size, int32_t global_q_offset, int32_t window, bool per_shard, int32_t tile_m,
              int32_t shard_base, int32_t total_shards) {
  Plan plan;
  if (total_shards <= 0) total_shards = shards;
  // key position of local token t of the call's shard r (its global index is shard_base + r)
  auto kpos = [&](int32_t r, int64_t t) {
    return kvp_position(shard_base + r, t, n_local, block_size, total_shards, mode);
  };
  const int64_t q_lo = global_q_offset, q_hi = (int64_t)global_q_offset + q_len - 1;
  std::vector<int32_t> shard_seg0(shards), shard_nseg(shards);
  for (int32_t r = 0; r < shards; ++r) {
    shard_seg0[r] = (int32_t)plan.segs.size();
    bool first = true;
    for (int32_t s0 = 0; s0 < n_local; s0 += seg_size) {
      const int32_t rows = std::min(seg_size, n_local - s0);
      const int64_t kmin = kpos(r, s0);
      const int64_t kmax = kpos(r, s0 + rows - 1);
      // drop segments no query can see (causal: kmin > last q; window: kmax too old for the first q)
      if (kmin > q_hi) continue;
      if (window > 0 && q_lo - kmax >= window && q_hi - kmax >= window) continue;
      plan.segs.push_back(Seg{s0, rows, 0, kSegCausal | (first ? kSegBlockStart : 0) | (r << kSegShardShift)});
      first = false;
    }
    shard_nseg[r] = (int32_t)plan.segs.size() - shard_seg0[r];
  }
  for (int32_t t0 = 0; t0 < q_len; t0 += tile_m) {
    const int32_t rows = std::min(tile_m, q_len - t0);
    const int32_t pos0 = global_q_offset + t0;
    for (int32_t r = 0; r < (per_shard ? shards : 1); ++r) {
      TileTask t{};
      t.row0 = t0;
      t.rows = rows;
      t.pos0 = pos0;
      t.seg0 = per_shard ? shard_seg0[r] : 0;
      t.nseg = per_shard ? shard_nseg[r] : (int32_t)plan.segs.size();
      t.aux = per_shard ? r : -1;
      t.head = 0;
      // weight: visible keys of the tile (every key position below the tile is one page of some shard;
      // this call holds shards / total_shards of them)
      int64_t lo = window > 0 ? std::max<int64_t>(0, pos0 - window + 1) : 0;
      int64_t span = (int64_t)pos0 + rows - lo;
      t.work = weight((int64_t)rows * span * shards / total_shards / (per_shard ? shards : 1));
      // where to cut the segment list for two halves of about equal work: count the 128-key
      // tiles of each segment this tile sees (the kernel's own skip rule)
      int64_t total = 0;
      std::vector<int64_t> seen(t.nseg);
      for (int32_t i = 0; i < t.nseg; ++i) {
        const Seg& g = plan.segs[t.seg0 + i];
        const int32_t r = g.flags >> kSegShardShift;
        int64_t n = 0;
        for (int32_t c0 = 0; c0 < g.rows; c0 += 128) {
          const int32_t nv = std::min(128, g.rows - c0);
          const int64_t kp0 = kpos(r, g.row0 + c0);
          const int64_t kp1 = kpos(r, g.row0 + c0 + nv - 1);
          if (kp0 > (int64_t)pos0 + rows - 1) continue;
          if (window > 0 && kp1 < (int64_t)pos0 - window + 1) continue;
          ++n;
        }
        seen[i] = n;
        total += n;
      }
      int64_t acc = 0;
      t.split1 = t.nseg > 1 ? 1 : t.nseg;
      for (int32_t i = 0; i + 1 < t.nseg; ++i) {
        acc += seen[i];
        t.split1 = i + 1;
        if (2 * acc >= total) break;
      }
      plan.tasks.push_back(t);
    }
  }
  expand_heads(plan, heads);
  return plan;
}

}  // namespace cbv
