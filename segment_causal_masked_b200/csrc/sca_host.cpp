// Host runtime of libsca: error state, the mask-metadata builder (per-token
// descriptors, block-sparse tile schedule, unmasked-pair count), the KV-cache
// object, metadata upload, and argument validation for the kernels.
//
// The visibility rule is the action-aware causal attention of the Hy-Nomas
// pages (picx.dev summary, Model Architecture, "Segment-wise Causal
// Attention" and "Action-Aware Causal Attention (Figure 6b)"; onedev.kr
// review, "무엇과 다른가"). Here it is evaluated as a predicate on descriptor
// words, the same predicate the attention kernel applies on PARTIAL tiles.

#include <math.h>

#include <cmath>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <numeric>
#include <queue>

#include "sca_camera.h"
#include "sca_internal.h"

namespace sca {

static thread_local std::string g_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_error = buf;
  return code;
}

int check_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return SCA_OK;
  return fail(SCA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool SegLayout::same(const SegLayout& o) const {
  if (F != o.F || G != o.G || h != o.h || n_act != o.n_act) return false;
  for (int a = 0; a < n_act; ++a)
    if (len[a] != o.len[a] || beg[a] != o.beg[a] || end[a] != o.end[a]) return false;
  return true;
}

int read_segment(const sca_segment* s, SegLayout* out) {
  if (!s) return fail(SCA_ERR_INVALID_ARG, "null segment");
  if (s->num_frames < 1 || s->tokens_per_frame < 1 || s->head_len < 0)
    return fail(SCA_ERR_INVALID_ARG,
                "segment needs num_frames >= 1, tokens_per_frame >= 1, head_len >= 0 "
                "(got %d, %d, %d)", s->num_frames, s->tokens_per_frame, s->head_len);
  if (s->num_actions < 0 || s->num_actions > SCA_MAX_ACTIONS)
    return fail(SCA_ERR_INVALID_ARG, "num_actions must be in [0, %d] (got %d)",
                SCA_MAX_ACTIONS, s->num_actions);
  if (s->num_actions > 0 && (!s->action_len || !s->action_begin || !s->action_end))
    return fail(SCA_ERR_INVALID_ARG, "null action arrays");
  SegLayout L;
  L.F = s->num_frames;
  L.G = s->tokens_per_frame;
  L.h = s->head_len;
  L.n_act = s->num_actions;
  for (int a = 0; a < L.n_act; ++a) {
    L.len[a] = s->action_len[a];
    L.beg[a] = s->action_begin[a];
    L.end[a] = s->action_end[a];
    if (L.len[a] < 1 || L.beg[a] < 0 || L.beg[a] >= L.end[a] || L.end[a] > L.F)
      return fail(SCA_ERR_INVALID_ARG,
                  "action %d needs length >= 1 and 0 <= begin < end <= num_frames "
                  "(got length %d, window [%d, %d), %d frames)",
                  a, L.len[a], L.beg[a], L.end[a], L.F);
  }
  if (L.n_tokens() > (int64_t(1) << 31) - 1)
    return fail(SCA_ERR_UNSUPPORTED, "segment has more than 2^31-1 tokens");
  *out = L;
  return SCA_OK;
}

uint32_t key_descriptor(const SegLayout& s, uint32_t seg, int64_t t) {
  const int64_t nv = s.n_video();
  if (t < nv) return seg | SCA_DESC_ALIVE;
  if (t < nv + s.h) return seg | SCA_DESC_ALIVE | SCA_DESC_HEAD;
  int64_t r = t - nv - s.h;
  int a = 0;
  while (a < s.n_act - 1 && r >= s.len[a]) r -= s.len[a++];
  return seg | SCA_DESC_TAIL | (uint32_t(a) << SCA_DESC_ACTION_SHIFT);
}

// The pair predicate: may a query described by (q0, q1) see key `k`?
// `window`: how many earlier segments a query may see (65535: all).
static inline bool visible(uint32_t q0, uint32_t q1, uint32_t k, uint32_t window) {
  if (!(q0 & SCA_QDESC_VALID)) return false;
  const uint32_t qs = q0 & SCA_DESC_SEG_MASK, ks = k & SCA_DESC_SEG_MASK;
  if (ks == qs)  // own segment: everything but the tails outside the query's set
    return !(k & SCA_DESC_TAIL) || ((q1 >> ((k >> SCA_DESC_ACTION_SHIFT) & 31u)) & 1u);
  // earlier segment inside the window: its live (video, head) keys, if the
  // query looks back
  return ks < qs && qs - ks <= window && (q0 & SCA_QDESC_SEES_PAST) && (k & SCA_DESC_ALIVE);
}

namespace {

// What one tile holds, enough to classify a (query tile, key tile) pair.
struct TileSummary {
  uint32_t seg_min = 0xFFFFFFFFu, seg_max = 0;
  bool oob = false;          // fewer than 128 existing rows
  bool all_flag = true;      // every row sees the past / every key alive
  bool any_flag = false;
  bool video_only = true;    // keys: no head or tail key in the tile
  std::vector<uint64_t> vals;  // distinct descriptors (query: q0 | q1 << 32)
  std::vector<int32_t> count;  // how many rows / keys carry each
  void add(uint64_t v, uint32_t seg, bool flag) {
    seg_min = std::min(seg_min, seg);
    seg_max = std::max(seg_max, seg);
    all_flag &= flag;
    any_flag |= flag;
    auto it = std::find(vals.begin(), vals.end(), v);
    if (it == vals.end()) {
      vals.push_back(v);
      count.push_back(1);
    } else {
      ++count[size_t(it - vals.begin())];
    }
  }
};

uint8_t classify(const TileSummary& q, const TileSummary& k, uint32_t window) {
  if (q.vals.empty() || k.vals.empty()) return SCA_TILE_EMPTY;
  if (k.seg_min > q.seg_max) return SCA_TILE_EMPTY;   // only later segments
  if (k.seg_max < q.seg_min) {                          // only earlier segments
    if (q.seg_min - k.seg_max > window) return SCA_TILE_EMPTY;  // all outside the window
    if (q.seg_max - k.seg_min <= window) {                      // all inside it
      if (!q.any_flag || !k.any_flag) return SCA_TILE_EMPTY;
      if (q.all_flag && k.all_flag && !q.oob && !k.oob) return SCA_TILE_FULL;
      return SCA_TILE_PARTIAL;
    }
  }
  bool any = false, all = !q.oob && !k.oob;
  for (uint64_t qv : q.vals)
    for (uint64_t kv : k.vals) {
      const bool v = visible(uint32_t(qv), uint32_t(qv >> 32), uint32_t(kv), window);
      any |= v;
      all &= v;
    }
  return !any ? SCA_TILE_EMPTY : (all ? SCA_TILE_FULL : SCA_TILE_PARTIAL);
}

}  // namespace

// Set by sca_set_split_override and read by the planners of the same host
// thread only, so a test or tuning loop on one thread cannot change the plan
// of a call another thread is making.
static thread_local int g_split_override = 0;

int split_override() { return g_split_override; }

// Limit of the kernels' pipeline waits for calls from this host thread
// (sca_set_pipeline_timeout_ns).
static thread_local unsigned long long g_pipeline_timeout_ns = 2000000000ull;

}  // namespace sca

using namespace sca;

extern "C" {

const char* sca_last_error(void) { return g_error.c_str(); }

int sca_metadata_create(sca_metadata** out) {
  if (!out) return fail(SCA_ERR_INVALID_ARG, "null output pointer");
  *out = new (std::nothrow) sca_metadata();
  return *out ? SCA_OK : fail(SCA_ERR_INVALID_ARG, "out of host memory");
}

void sca_metadata_destroy(sca_metadata* md) {
  if (!md) return;
  if (md->upload_done) {
    cudaEventSynchronize(md->upload_done);
    cudaEventDestroy(md->upload_done);
  }
  if (md->dev) cudaFree(md->dev);
  if (md->pinned) cudaFreeHost(md->pinned);
  delete md;
}

int sca_build_segment_mask_metadata(sca_metadata* md, const sca_segment* cached,
                                    int32_t n_cached, const sca_segment* current,
                                    int32_t n_current, int32_t policy) {
  sca_mask_options opt;
  memset(&opt, 0, sizeof(opt));
  opt.textq_policy = policy;
  opt.history_segments = -1;
  return sca_build_segment_mask_metadata_ex(md, cached, n_cached, current, n_current, &opt);
}

int sca_build_segment_mask_metadata_ex(sca_metadata* md, const sca_segment* cached,
                                       int32_t n_cached, const sca_segment* current,
                                       int32_t n_current, const sca_mask_options* opt) {
  const int32_t policy = opt ? opt->textq_policy : SCA_TEXTQ_OWN_TAIL;
  const uint32_t window = (opt && opt->history_segments >= 0)
                              ? uint32_t(std::min(opt->history_segments, 65535)) : 65535u;
  const uint8_t* keep = opt ? opt->keep_blocks : nullptr;
  if (!md) return fail(SCA_ERR_INVALID_ARG, "null metadata handle");
  if (n_cached < 0 || n_current < 1)
    return fail(SCA_ERR_INVALID_ARG, "need n_cached >= 0 and n_current >= 1");
  if (int64_t(n_cached) + n_current > SCA_MAX_SEGMENTS)
    return fail(SCA_ERR_UNSUPPORTED, "more than %d segments", SCA_MAX_SEGMENTS);
  if ((n_cached > 0 && !cached) || !current)
    return fail(SCA_ERR_INVALID_ARG, "null segment array");
  if (policy != SCA_TEXTQ_OWN_TAIL && policy != SCA_TEXTQ_FULL_SEGMENT)
    return fail(SCA_ERR_INVALID_ARG, "unknown text-query policy %d", policy);

  std::vector<SegLayout> segs((size_t)n_cached + n_current);
  for (int i = 0; i < n_cached; ++i) {
    int rc = read_segment(&cached[i], &segs[i]);
    if (rc) return rc;
  }
  for (int j = 0; j < n_current; ++j) {
    int rc = read_segment(&current[j], &segs[size_t(n_cached) + j]);
    if (rc) return rc;
  }
  int64_t n_cache = 0, n_q = 0;
  for (int i = 0; i < n_cached; ++i) n_cache += segs[i].n_tokens();
  for (int j = 0; j < n_current; ++j) n_q += segs[size_t(n_cached) + j].n_tokens();
  if (n_cache > (int64_t(1) << 31) - 1 || n_q > (int64_t(1) << 31) - 256)
    return fail(SCA_ERR_UNSUPPORTED, "more than 2^31 keys or queries");
  const int64_t n_ct = (n_cache + SCA_TILE - 1) / SCA_TILE;
  const int64_t n_ut = (n_q + SCA_TILE - 1) / SCA_TILE;
  if (n_ct + n_ut > int64_t(kPairTileMask))
    return fail(SCA_ERR_UNSUPPORTED, "more than 2^24 key tiles");

  // --- descriptors ---------------------------------------------------------
  std::vector<uint32_t> kdesc_cache((size_t)n_cache);
  {
    int64_t pos = 0;
    for (int i = 0; i < n_cached; ++i)
      for (int64_t t = 0; t < segs[i].n_tokens(); ++t)
        kdesc_cache[size_t(pos++)] = key_descriptor(segs[i], uint32_t(i), t);
  }
  std::vector<uint32_t> kdesc_cur((size_t)n_q), qdesc((size_t)(2 * n_q));
  int64_t A = 0;
  {
    // alive keys of all earlier segments, for A
    std::vector<int64_t> alive_before(segs.size() + 1, 0);
    for (size_t s = 0; s < segs.size(); ++s)
      alive_before[s + 1] = alive_before[s] + segs[s].n_video() + segs[s].h;
    const bool full = policy == SCA_TEXTQ_FULL_SEGMENT;
    int64_t q = 0;
    for (int j = 0; j < n_current; ++j) {
      const uint32_t g = uint32_t(n_cached + j);
      const SegLayout& S = segs[g];
      const int64_t own_live = S.n_video() + S.h;
      auto emit = [&](int64_t count, uint32_t w0, uint32_t w1) {
        const int64_t first = std::max<int64_t>(0, int64_t(g) - int64_t(window));  // oldest visible
        int64_t seen = own_live + ((w0 & SCA_QDESC_SEES_PAST)
                                       ? alive_before[g] - alive_before[size_t(first)] : 0);
        for (int a = 0; a < S.n_act; ++a)
          if ((w1 >> a) & 1u) seen += S.len[a];
        A += count * seen;
        for (int64_t i = 0; i < count; ++i, ++q) {
          qdesc[size_t(2 * q)] = w0;
          qdesc[size_t(2 * q + 1)] = w1;
        }
      };
      const uint32_t base = g | SCA_QDESC_VALID;
      for (int f = 0; f < S.F; ++f) emit(S.G, base | SCA_QDESC_SEES_PAST, S.frame_mask(f));
      const uint32_t text0 = base | (full ? SCA_QDESC_SEES_PAST : 0u);
      emit(S.h, text0, full ? S.all_actions() : 0u);
      for (int a = 0; a < S.n_act; ++a) emit(S.len[a], text0, full ? S.all_actions() : (1u << a));
    }
    int64_t pos = 0;
    for (int j = 0; j < n_current; ++j) {
      const uint32_t g = uint32_t(n_cached + j);
      for (int64_t t = 0; t < segs[g].n_tokens(); ++t)
        kdesc_cur[size_t(pos++)] = key_descriptor(segs[g], g, t);
    }
  }

  // --- tile summaries ------------------------------------------------------
  const int n_qt = int((n_q + SCA_TILE - 1) / SCA_TILE);
  std::vector<TileSummary> qs((size_t)n_qt), ks((size_t)(n_ct + n_ut));
  for (int64_t i = 0; i < n_q; ++i) {
    const uint32_t w0 = qdesc[size_t(2 * i)], w1 = qdesc[size_t(2 * i + 1)];
    qs[size_t(i / SCA_TILE)].add(uint64_t(w0) | (uint64_t(w1) << 32), w0 & SCA_DESC_SEG_MASK,
                                 (w0 & SCA_QDESC_SEES_PAST) != 0);
  }
  qs[size_t(n_qt - 1)].oob = (n_q % SCA_TILE) != 0;
  auto add_keys = [&](const std::vector<uint32_t>& d, int64_t n, int64_t tile0) {
    for (int64_t i = 0; i < n; ++i) {
      TileSummary& K = ks[size_t(tile0 + i / SCA_TILE)];
      K.add(d[size_t(i)], d[size_t(i)] & SCA_DESC_SEG_MASK, (d[size_t(i)] & SCA_DESC_ALIVE) != 0);
      if (d[size_t(i)] & (SCA_DESC_HEAD | SCA_DESC_TAIL)) K.video_only = false;
    }
    if (n % SCA_TILE) ks[size_t(tile0 + n / SCA_TILE)].oob = true;
  };
  add_keys(kdesc_cache, n_cache, 0);
  add_keys(kdesc_cur, n_q, n_ct);
  const int64_t n_kt = n_ct + n_ut;
  if (keep && (opt->keep_blocks_len != int64_t(n_qt) * n_kt))
    return fail(SCA_ERR_INVALID_ARG, "keep_blocks has %lld entries, the layout has %d x %lld tiles",
                (long long)opt->keep_blocks_len, n_qt, (long long)n_kt);

  // --- runs of equal descriptors inside each key tile (for the kernel's
  // per-row visibility masks on PARTIAL tiles, and to count dropped pairs) --
  std::vector<int32_t> run_ptr(size_t(n_kt) + 1, 0);
  std::vector<uint32_t> runs;
  auto add_runs = [&](const std::vector<uint32_t>& d, int64_t n, int64_t tile0) {
    for (int64_t t = 0; t * SCA_TILE < n; ++t) {
      const int64_t k0 = t * SCA_TILE, k1 = std::min<int64_t>(n, k0 + SCA_TILE);
      int64_t a = k0;
      while (a < k1) {
        int64_t b = a + 1;
        while (b < k1 && d[size_t(b)] == d[size_t(a)]) ++b;
        runs.push_back(uint32_t(a - k0) | (uint32_t(b - a) << 8));
        runs.push_back(d[size_t(a)]);
        a = b;
      }
      run_ptr[size_t(tile0 + t) + 1] = int32_t(runs.size() / 2);
    }
  };
  add_runs(kdesc_cache, n_cache, 0);
  add_runs(kdesc_cur, n_q, n_ct);
  // visible (query, key) pairs of one tile pair, for blocks that are dropped
  auto block_pairs = [&](const TileSummary& Q, int64_t kt) {
    int64_t n = 0;
    for (size_t a = 0; a < Q.vals.size(); ++a)
      for (int32_t r = run_ptr[size_t(kt)]; r < run_ptr[size_t(kt) + 1]; ++r)
        if (visible(uint32_t(Q.vals[a]), uint32_t(Q.vals[a] >> 32), runs[size_t(2 * r + 1)], window))
          n += int64_t(Q.count[a]) * int64_t((runs[size_t(2 * r)] >> 8) & 255u);
    return n;
  };

  // --- classification and CSR ---------------------------------------------
  std::vector<int32_t> row_ptr(size_t(n_qt) + 1, 0), kv_tile;
  std::vector<uint8_t> flag;
  int64_t n_full = 0, n_partial = 0, n_dropped = 0;
  kv_tile.reserve(size_t(n_qt) * 64);
  flag.reserve(size_t(n_qt) * 64);
  for (int qt = 0; qt < n_qt; ++qt) {
    const TileSummary& Q = qs[size_t(qt)];
    for (int64_t kt = 0; kt < n_ct + n_ut; ++kt) {
      const TileSummary& K = ks[size_t(kt)];
      if (kt < n_ct && K.seg_min > Q.seg_max) { kt = n_ct - 1; continue; }  // rest of cache is later
      if (kt >= n_ct && K.seg_min > Q.seg_max) break;
      const uint8_t c = classify(Q, K, window);
      if (c == SCA_TILE_EMPTY) continue;
      if (keep && !keep[size_t(qt) * size_t(n_kt) + size_t(kt)] && K.video_only) {
        A -= block_pairs(Q, kt);  // a dropped video block
        ++n_dropped;
        continue;
      }
      kv_tile.push_back(int32_t(kt));
      flag.push_back(c);
      (c == SCA_TILE_FULL ? n_full : n_partial) += 1;
    }
    row_ptr[size_t(qt) + 1] = int32_t(kv_tile.size());
    if (kv_tile.size() > size_t(INT32_MAX) - 4096)
      return fail(SCA_ERR_UNSUPPORTED, "schedule larger than 2^31 entries");
  }

  // --- kernel work list: query-tile pairs, union of their key tiles --------
  const int n_pairs = (n_qt + 1) / 2;
  std::vector<int32_t> pair_ptr(size_t(n_pairs) + 1, 0);
  std::vector<uint32_t> pair_list;
  pair_list.reserve(kv_tile.size());
  for (int p = 0; p < n_pairs; ++p) {
    const int a = 2 * p, b = 2 * p + 1;
    int32_t ia = row_ptr[size_t(a)], ea = row_ptr[size_t(a) + 1];
    int32_t ib = b < n_qt ? row_ptr[size_t(b)] : 0, eb = b < n_qt ? row_ptr[size_t(b) + 1] : 0;
    while (ia < ea || ib < eb) {
      const int32_t ta = ia < ea ? kv_tile[size_t(ia)] : INT32_MAX;
      const int32_t tb = ib < eb ? kv_tile[size_t(ib)] : INT32_MAX;
      const int32_t t = std::min(ta, tb);
      uint32_t e = uint32_t(t);
      if (ta == t) e |= uint32_t(flag[size_t(ia++)]) << 24;
      if (tb == t) e |= uint32_t(flag[size_t(ib++)]) << 26;
      pair_list.push_back(e);
    }
    pair_ptr[size_t(p) + 1] = int32_t(pair_list.size());
  }
  // Estimated cost of a pair, in (query tile x key tile) units: a FULL tile
  // is one unit, a PARTIAL one a little more (its mask), an EMPTY one only
  // the shared loads and handshakes (the kernel skips its MMAs and softmax).
  std::vector<float> pair_cost((size_t)n_pairs, 0.f);
  const float w_cls[4] = {0.1f, 1.25f, 1.f, 0.f};
  for (int p = 0; p < n_pairs; ++p) {
    float c = 0.f;
    for (int32_t i = pair_ptr[size_t(p)]; i < pair_ptr[size_t(p) + 1]; ++i)
      c += w_cls[(pair_list[size_t(i)] >> 24) & 3u] + w_cls[(pair_list[size_t(i)] >> 26) & 3u];
    pair_cost[size_t(p)] = c;
  }
  std::vector<int32_t> order((size_t)n_pairs);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int32_t x, int32_t y) {
    return pair_cost[size_t(x)] > pair_cost[size_t(y)];
  });

  // --- backward work lists (layouts without a cache: keys = queries) ------
  // per key tile, the query tiles that see it (the transposed schedule),
  // longest list first; per query tile, runs of equal query descriptors; the
  // key descriptors padded to whole tiles.
  std::vector<int32_t> kt_ptr, kt_order, qrun_ptr;
  std::vector<uint32_t> kt_list, qruns, kdesc_pad;
  if (n_cached == 0) {
    const int n_kt = int(n_ut);
    kt_ptr.assign(size_t(n_kt) + 1, 0);
    for (int32_t t : kv_tile) kt_ptr[size_t(t - n_ct) + 1] += 1;
    for (int t = 0; t < n_kt; ++t) kt_ptr[size_t(t) + 1] += kt_ptr[size_t(t)];
    kt_list.resize(kv_tile.size());
    std::vector<int32_t> pos(kt_ptr.begin(), kt_ptr.end() - 1);
    for (int qt = 0; qt < n_qt; ++qt)
      for (int32_t i = row_ptr[size_t(qt)]; i < row_ptr[size_t(qt) + 1]; ++i)
        kt_list[size_t(pos[size_t(kv_tile[size_t(i)] - n_ct)]++)] =
            uint32_t(qt) | (uint32_t(flag[size_t(i)]) << 24);
    std::vector<float> kt_cost(size_t(n_kt), 0.f);
    for (int t = 0; t < n_kt; ++t)
      for (int32_t i = kt_ptr[size_t(t)]; i < kt_ptr[size_t(t) + 1]; ++i)
        kt_cost[size_t(t)] += w_cls[(kt_list[size_t(i)] >> 24) & 3u];
    kt_order.resize(size_t(n_kt));
    std::iota(kt_order.begin(), kt_order.end(), 0);
    std::stable_sort(kt_order.begin(), kt_order.end(), [&](int32_t x, int32_t y) {
      return kt_cost[size_t(x)] > kt_cost[size_t(y)];
    });
    qrun_ptr.assign(size_t(n_qt) + 1, 0);
    for (int qt = 0; qt < n_qt; ++qt) {
      const int64_t r0 = int64_t(qt) * SCA_TILE, r1 = std::min<int64_t>(n_q, r0 + SCA_TILE);
      for (int64_t a = r0; a < r1;) {
        int64_t b = a + 1;
        while (b < r1 && qdesc[size_t(2 * b)] == qdesc[size_t(2 * a)] &&
               qdesc[size_t(2 * b + 1)] == qdesc[size_t(2 * a + 1)])
          ++b;
        qruns.push_back(uint32_t(a - r0) | (uint32_t(b - a) << 8));
        qruns.push_back(qdesc[size_t(2 * a)]);
        qruns.push_back(qdesc[size_t(2 * a + 1)]);
        qruns.push_back(0u);
        a = b;
      }
      qrun_ptr[size_t(qt) + 1] = int32_t(qruns.size() / 4);
    }
    kdesc_pad.assign(size_t(n_qt) * SCA_TILE, 0u);
    std::copy(kdesc_cur.begin(), kdesc_cur.end(), kdesc_pad.begin());
  }

  md->built = true;
  md->uploaded = false;
  md->plan_key[0] = -1;
  md->n_cached = n_cached;
  md->n_current = n_current;
  md->policy = policy;
  md->history = int32_t(window);
  md->n_dropped = n_dropped;
  md->segs.swap(segs);
  md->n_cache = n_cache;
  md->n_q = n_q;
  md->unmasked_pairs = A;
  md->n_q_tiles = n_qt;
  md->n_cache_tiles = int32_t(n_ct);
  md->n_kv_tiles = int32_t(n_ct + n_ut);
  md->n_pairs = n_pairs;
  md->n_full = n_full;
  md->n_partial = n_partial;
  md->key_desc_cur.swap(kdesc_cur);
  md->query_desc.swap(qdesc);
  md->row_ptr.swap(row_ptr);
  md->kv_tile.swap(kv_tile);
  md->flag.swap(flag);
  md->pair_ptr.swap(pair_ptr);
  md->pair_list.swap(pair_list);
  md->item_order.swap(order);
  md->pair_cost.swap(pair_cost);
  md->run_ptr.swap(run_ptr);
  md->runs.swap(runs);
  md->kt_ptr.swap(kt_ptr);
  md->kt_list.swap(kt_list);
  md->kt_order.swap(kt_order);
  md->qrun_ptr.swap(qrun_ptr);
  md->qruns.swap(qruns);
  md->kdesc_pad.swap(kdesc_pad);
  return SCA_OK;
}

int sca_metadata_get_counts(const sca_metadata* md, int64_t* unmasked_pairs, int64_t* n_queries,
                            int64_t* n_cache_keys, int32_t* n_q_tiles, int32_t* n_kv_tiles,
                            int64_t* nnz, int64_t* n_full, int64_t* n_partial) {
  if (!md || !md->built) return fail(SCA_ERR_INVALID_ARG, "metadata not built");
  if (unmasked_pairs) *unmasked_pairs = md->unmasked_pairs;
  if (n_queries) *n_queries = md->n_q;
  if (n_cache_keys) *n_cache_keys = md->n_cache;
  if (n_q_tiles) *n_q_tiles = md->n_q_tiles;
  if (n_kv_tiles) *n_kv_tiles = md->n_kv_tiles;
  if (nnz) *nnz = int64_t(md->kv_tile.size());
  if (n_full) *n_full = md->n_full;
  if (n_partial) *n_partial = md->n_partial;
  return SCA_OK;
}

int sca_metadata_get_schedule(const sca_metadata* md, const int32_t** row_ptr,
                              const int32_t** kv_tile, const uint8_t** flag) {
  if (!md || !md->built) return fail(SCA_ERR_INVALID_ARG, "metadata not built");
  if (row_ptr) *row_ptr = md->row_ptr.data();
  if (kv_tile) *kv_tile = md->kv_tile.data();
  if (flag) *flag = md->flag.data();
  return SCA_OK;
}

int sca_metadata_get_descriptors(const sca_metadata* md, const uint32_t** key_desc,
                                 const uint32_t** query_desc) {
  if (!md || !md->built) return fail(SCA_ERR_INVALID_ARG, "metadata not built");
  if (key_desc) *key_desc = md->key_desc_cur.data();
  if (query_desc) *query_desc = md->query_desc.data();
  return SCA_OK;
}

int sca_metadata_get_bwd_schedule(const sca_metadata* md, const int32_t** kt_ptr,
                                  const uint32_t** kt_list, const int32_t** kt_order) {
  if (!md || !md->built) return fail(SCA_ERR_INVALID_ARG, "metadata not built");
  const bool has = !md->kt_ptr.empty();  // NULL outputs for a layout with a cache
  if (kt_ptr) *kt_ptr = has ? md->kt_ptr.data() : nullptr;
  if (kt_list) *kt_list = has ? md->kt_list.data() : nullptr;
  if (kt_order) *kt_order = has ? md->kt_order.data() : nullptr;
  return SCA_OK;
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int sca_metadata_upload(sca_metadata* md, void* stream) {
  if (!md || !md->built) return fail(SCA_ERR_INVALID_ARG, "metadata not built");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0;
  if (int rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice")) return rc;
  // layout of the device block
  const size_t nq_pad = size_t(md->n_pairs) * 2 * SCA_TILE;
  size_t off = 0;
  const size_t off_q = off;     off = align_up(off + nq_pad * 8, 256);
  const size_t off_o = off;     off = align_up(off + size_t(md->n_pairs) * 4, 256);
  const size_t off_p = off;     off = align_up(off + (size_t(md->n_pairs) + 1) * 4, 256);
  const size_t off_l = off;     off = align_up(off + std::max<size_t>(md->pair_list.size(), 1) * 4, 256);
  const size_t off_rp = off;    off = align_up(off + md->run_ptr.size() * 4, 256);
  const size_t off_r = off;     off = align_up(off + std::max<size_t>(md->runs.size(), 2) * 4, 256);
  // backward lists (empty unless the layout has no cache)
  const size_t off_ktp = off;   off = align_up(off + md->kt_ptr.size() * 4, 256);
  const size_t off_ktl = off;   off = align_up(off + md->kt_list.size() * 4, 256);
  const size_t off_kto = off;   off = align_up(off + md->kt_order.size() * 4, 256);
  const size_t off_qrp = off;   off = align_up(off + md->qrun_ptr.size() * 4, 256);
  const size_t off_qr = off;    off = align_up(off + md->qruns.size() * 4, 256);
  const size_t off_kd = off;    off = align_up(off + md->kdesc_pad.size() * 4, 256);
  const size_t bytes = off;

  if (md->upload_done) {  // the staging buffer may still feed the previous copy
    if (int rc = check_cuda(cudaEventSynchronize(md->upload_done), "cudaEventSynchronize")) return rc;
  } else if (int rc = check_cuda(cudaEventCreateWithFlags(&md->upload_done, cudaEventDisableTiming),
                                 "cudaEventCreate")) {
    return rc;
  }
  if (md->dev && (md->device != dev || md->dev_bytes < bytes)) {
    cudaFree(md->dev);
    md->dev = nullptr;
    md->dev_bytes = 0;
  }
  if (!md->dev) {
    if (int rc = check_cuda(cudaMalloc(&md->dev, bytes), "cudaMalloc(metadata)")) return rc;
    md->dev_bytes = bytes;
    md->device = dev;
  }
  if (md->pinned_bytes < bytes) {
    if (md->pinned) cudaFreeHost(md->pinned);
    md->pinned = nullptr;
    md->pinned_bytes = 0;
    if (int rc = check_cuda(cudaMallocHost(&md->pinned, bytes), "cudaMallocHost(metadata)")) return rc;
    md->pinned_bytes = bytes;
  }
  uint8_t* h = static_cast<uint8_t*>(md->pinned);
  memset(h, 0, bytes);
  memcpy(h + off_q, md->query_desc.data(), md->query_desc.size() * 4);  // padding: invalid queries
  memcpy(h + off_o, md->item_order.data(), md->item_order.size() * 4);
  memcpy(h + off_p, md->pair_ptr.data(), md->pair_ptr.size() * 4);
  memcpy(h + off_l, md->pair_list.data(), md->pair_list.size() * 4);
  memcpy(h + off_rp, md->run_ptr.data(), md->run_ptr.size() * 4);
  memcpy(h + off_r, md->runs.data(), md->runs.size() * 4);
  memcpy(h + off_ktp, md->kt_ptr.data(), md->kt_ptr.size() * 4);
  memcpy(h + off_ktl, md->kt_list.data(), md->kt_list.size() * 4);
  memcpy(h + off_kto, md->kt_order.data(), md->kt_order.size() * 4);
  memcpy(h + off_qrp, md->qrun_ptr.data(), md->qrun_ptr.size() * 4);
  memcpy(h + off_qr, md->qruns.data(), md->qruns.size() * 4);
  memcpy(h + off_kd, md->kdesc_pad.data(), md->kdesc_pad.size() * 4);
  if (int rc = check_cuda(cudaMemcpyAsync(md->dev, h, bytes, cudaMemcpyHostToDevice, st),
                          "cudaMemcpyAsync(metadata)"))
    return rc;
  if (int rc = check_cuda(cudaEventRecord(md->upload_done, st), "cudaEventRecord")) return rc;
  md->off_qdesc = off_q;
  md->off_order = off_o;
  md->off_ptr = off_p;
  md->off_list = off_l;
  md->off_run_ptr = off_rp;
  md->off_runs = off_r;
  md->off_kt_ptr = off_ktp;
  md->off_kt_list = off_ktl;
  md->off_kt_order = off_kto;
  md->off_qrun_ptr = off_qrp;
  md->off_qruns = off_qr;
  md->off_kdesc = off_kd;
  md->uploaded = true;
  return SCA_OK;
}

// ---------------------------------------------------------------------------
// KV cache
// ---------------------------------------------------------------------------

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sca_kv_cache_create(sca_kv_cache** out, int32_t heads, int32_t head_dim, int64_t capacity,
                        void* k_buf, void* v_buf, void* desc_buf) {
  if (!out) return fail(SCA_ERR_INVALID_ARG, "null output pointer");
  *out = nullptr;
  if (head_dim != SCA_HEAD_DIM) return fail(SCA_ERR_UNSUPPORTED, "head_dim must be 128");
  if (heads < 1 || capacity < 1 || capacity > (int64_t(1) << 31) - 1)
    return fail(SCA_ERR_INVALID_ARG, "need heads >= 1 and 1 <= capacity < 2^31");
  if (!k_buf || !v_buf || !desc_buf) return fail(SCA_ERR_INVALID_ARG, "null cache buffer");
  if (!aligned16(k_buf) || !aligned16(v_buf) || !aligned16(desc_buf))
    return fail(SCA_ERR_MISALIGNED, "cache buffers must be 16-byte aligned");
  sca_kv_cache* c = new (std::nothrow) sca_kv_cache();
  if (!c) return fail(SCA_ERR_INVALID_ARG, "out of host memory");
  c->heads = heads;
  c->capacity = capacity;
  c->k = k_buf;
  c->v = v_buf;
  c->desc = static_cast<uint32_t*>(desc_buf);
  *out = c;
  return SCA_OK;
}

int sca_kv_cache_create_int8(sca_kv_cache** out, int32_t heads, int32_t head_dim,
                             int64_t capacity, void* k_codes, void* v_codes, float* k_scale,
                             float* v_scale, void* desc_buf) {
  if (!out) return fail(SCA_ERR_INVALID_ARG, "null output pointer");
  *out = nullptr;
  if (head_dim != SCA_HEAD_DIM) return fail(SCA_ERR_UNSUPPORTED, "head_dim must be 128");
  if (heads < 1 || capacity < 1 || capacity > (int64_t(1) << 31) - 1)
    return fail(SCA_ERR_INVALID_ARG, "need heads >= 1 and 1 <= capacity < 2^31");
  if (capacity % 4)
    return fail(SCA_ERR_INVALID_ARG, "an INT8 cache needs a capacity that is a multiple of 4 (got %lld)",
                (long long)capacity);
  if (!k_codes || !v_codes || !k_scale || !v_scale || !desc_buf)
    return fail(SCA_ERR_INVALID_ARG, "null cache buffer");
  if (!aligned16(k_codes) || !aligned16(v_codes) || !aligned16(k_scale) || !aligned16(v_scale) ||
      !aligned16(desc_buf))
    return fail(SCA_ERR_MISALIGNED, "cache buffers must be 16-byte aligned");
  sca_kv_cache* c = new (std::nothrow) sca_kv_cache();
  if (!c) return fail(SCA_ERR_INVALID_ARG, "out of host memory");
  c->heads = heads;
  c->capacity = capacity;
  c->int8 = true;
  c->k = k_codes;
  c->v = v_codes;
  c->k_scale = k_scale;
  c->v_scale = v_scale;
  c->desc = static_cast<uint32_t*>(desc_buf);
  *out = c;
  return SCA_OK;
}

void sca_kv_cache_destroy(sca_kv_cache* c) { delete c; }

int sca_kv_cache_get(const sca_kv_cache* c, int64_t* length, int32_t* n_segments) {
  if (!c) return fail(SCA_ERR_INVALID_ARG, "null cache");
  if (length) *length = c->length;
  if (n_segments) *n_segments = int32_t(c->segs.size());
  return SCA_OK;
}

int sca_kv_cache_truncate(sca_kv_cache* c, int32_t n_segments) {
  if (!c) return fail(SCA_ERR_INVALID_ARG, "null cache");
  if (n_segments < 0 || size_t(n_segments) > c->segs.size())
    return fail(SCA_ERR_INVALID_ARG, "cache holds %zu segments, cannot keep %d",
                c->segs.size(), n_segments);
  c->length = n_segments == 0 ? 0 : c->seg_start[size_t(n_segments)];
  c->segs.resize(size_t(n_segments));
  c->seg_start.resize(size_t(n_segments) + 1);
  return SCA_OK;
}

int sca_kv_cache_append(sca_kv_cache* c, const sca_segment* segment, const void* k,
                        const void* v, void* stream) {
  if (!c) return fail(SCA_ERR_INVALID_ARG, "null cache");
  SegLayout L;
  if (int rc = read_segment(segment, &L)) return rc;
  if (!k || !v) return fail(SCA_ERR_INVALID_ARG, "null k or v");
  if (!aligned16(k) || !aligned16(v)) return fail(SCA_ERR_MISALIGNED, "k and v must be 16-byte aligned");
  if (c->segs.size() >= SCA_MAX_SEGMENTS - 1)
    return fail(SCA_ERR_UNSUPPORTED, "cache already holds %zu segments", c->segs.size());
  const int64_t n = L.n_tokens();
  if (c->length + n > c->capacity)
    return fail(SCA_ERR_CAPACITY, "cache of capacity %lld holds %lld keys; segment of %lld does not fit",
                (long long)c->capacity, (long long)c->length, (long long)n);
  AppendArgs a{};
  a.k = k;
  a.v = v;
  a.k_cache = c->k;
  a.v_cache = c->v;
  a.k_scale = c->k_scale;
  a.v_scale = c->v_scale;
  a.int8 = c->int8 ? 1 : 0;
  a.desc = c->desc;
  a.length = c->length;
  a.capacity = c->capacity;
  a.n = int32_t(n);
  a.heads = c->heads;
  a.seg_index = uint32_t(c->segs.size());
  a.n_video = int32_t(L.n_video());
  a.head_len = L.h;
  a.n_act = L.n_act;
  a.tail_start[0] = 0;
  for (int i = 0; i < L.n_act; ++i) a.tail_start[i + 1] = a.tail_start[i] + L.len[i];
  if (int rc = check_cuda(launch_append(a, static_cast<cudaStream_t>(stream)), "kv_cache_append launch"))
    return rc;
  if (c->seg_start.empty()) c->seg_start.push_back(0);
  c->segs.push_back(L);
  c->length += n;
  c->seg_start.push_back(c->length);
  return SCA_OK;
}

// ---------------------------------------------------------------------------
// attention
// ---------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Looked up once (a function-local static is initialised exactly once, also
// when several host threads get here at the same time).
static EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return nullptr;
  }();
  return fn;
}

// bf16 tensor of rows of 128 elements, viewed as 3-D (128, dim1, dim2) with the
// given byte strides of dims 1 and 2; box (64, box1, box2), 128-byte swizzle.
static int make_map(CUtensorMap* m, const void* base, uint64_t dim1, uint64_t dim2,
                    uint64_t stride1, uint64_t stride2, uint32_t box1, uint32_t box2) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(SCA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[3] = {SCA_HEAD_DIM, dim1, dim2};
  cuuint64_t strides[2] = {stride1, stride2};
  cuuint32_t box[3] = {64, box1, box2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SCA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return SCA_OK;
}

// INT8 cache codes [heads][capacity][128] viewed as 3-D (128 bytes, rows,
// heads); box (128, 128, 1), 128-byte swizzle (one box row is one swizzle
// span). Rows at and past `rows` read as zeros.
static int make_code_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t heads,
                         uint64_t capacity) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(SCA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[3] = {SCA_HEAD_DIM, rows, heads};
  cuuint64_t strides[2] = {SCA_HEAD_DIM, capacity * SCA_HEAD_DIM};
  cuuint32_t box[3] = {SCA_HEAD_DIM, SCA_TILE, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SCA_ERR_CUDA, "cuTensorMapEncodeTiled (codes) failed (%d)", int(r));
  return SCA_OK;
}

// INT8 cache scales [heads][capacity] fp32 as 2-D (rows, heads); box (128, 1).
static int make_scale_map(CUtensorMap* m, const float* base, uint64_t rows, uint64_t heads,
                          uint64_t capacity) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(SCA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[2] = {rows, heads};
  cuuint64_t strides[1] = {capacity * 4};
  cuuint32_t box[2] = {SCA_TILE, 1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SCA_ERR_CUDA, "cuTensorMapEncodeTiled (scales) failed (%d)", int(r));
  return SCA_OK;
}

// ---------------------------------------------------------------------------
// camera cross-attention
// ---------------------------------------------------------------------------

int sca_camera_cross_attn(const void* q, const int32_t* q_frame, const void* k_cam,
                          const void* v_cam, const void* x, void* out, int32_t n_q, int32_t n_cam,
                          int32_t heads, int32_t mode, float softmax_scale, int32_t* dev_status,
                          void* stream) {
  if (n_q < 0 || heads < 1) return fail(SCA_ERR_INVALID_ARG, "n_q must be >= 0 and heads >= 1");
  if (n_cam < 1 || n_cam > SCA_MAX_CAMERA_TOKENS)
    return fail(SCA_ERR_INVALID_ARG, "n_cam must be in [1, %d]", SCA_MAX_CAMERA_TOKENS);
  if (mode != SCA_CAM_ALL && mode != SCA_CAM_OWN_FRAME && mode != SCA_CAM_UP_TO_FRAME)
    return fail(SCA_ERR_INVALID_ARG, "unknown camera attention mode %d", mode);
  if (!std::isfinite(softmax_scale)) return fail(SCA_ERR_INVALID_ARG, "softmax_scale must be finite");
  if (int64_t(n_q) * heads > INT32_MAX / 128 || heads > 65535)
    return fail(SCA_ERR_UNSUPPORTED, "too many query rows or heads");
  if (!k_cam || !v_cam) return fail(SCA_ERR_INVALID_ARG, "null camera keys or values");
  if (!aligned16(k_cam) || !aligned16(v_cam))
    return fail(SCA_ERR_MISALIGNED, "camera keys and values must be 16-byte aligned");
  if (n_q > 0) {
    if (!q || !x || !out) return fail(SCA_ERR_INVALID_ARG, "null q, x or out");
    if (!aligned16(q) || !aligned16(x) || !aligned16(out))
      return fail(SCA_ERR_MISALIGNED, "q, x and out must be 16-byte aligned");
    if (mode != SCA_CAM_ALL && !q_frame)
      return fail(SCA_ERR_INVALID_ARG, "the frame modes need q_frame");
    // out may be x itself; any other overlap of out with an input is refused
    const uint64_t bytes = uint64_t(n_q) * uint64_t(heads) * SCA_HEAD_DIM * 2;
    auto overlaps = [&](const void* p, uint64_t n) {
      const uintptr_t a0 = reinterpret_cast<uintptr_t>(out), b0 = reinterpret_cast<uintptr_t>(p);
      return a0 < b0 + n && b0 < a0 + bytes;
    };
    const uint64_t cam_bytes = uint64_t(n_cam) * uint64_t(heads) * SCA_HEAD_DIM * 2;
    if ((out != x && overlaps(x, bytes)) || overlaps(q, bytes) || overlaps(k_cam, cam_bytes) ||
        overlaps(v_cam, cam_bytes))
      return fail(SCA_ERR_INVALID_ARG, "out overlaps an input (only out == x is allowed)");
  }
  CamArgs a{};
  a.q_frame = mode == SCA_CAM_ALL ? nullptr : q_frame;
  a.n_q = n_q;
  a.n_cam = n_cam;
  a.heads = heads;
  a.mode = mode;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.status = dev_status;
  a.timeout_ns = g_pipeline_timeout_ns;
  if (n_q == 0) return SCA_OK;
  CamMaps maps;
  const uint64_t row = uint64_t(heads) * SCA_HEAD_DIM * 2;
  const uint32_t box = uint32_t(camera_box_rows(n_cam));
  int rc = make_map(&maps.q, q, uint64_t(heads), uint64_t(n_q), SCA_HEAD_DIM * 2, row, 1, 128);
  if (!rc) rc = make_map(&maps.x, x, uint64_t(heads), uint64_t(n_q), SCA_HEAD_DIM * 2, row, 1, 128);
  if (!rc) rc = make_map(&maps.out, out, uint64_t(heads), uint64_t(n_q), SCA_HEAD_DIM * 2, row, 1, 128);
  if (!rc) rc = make_map(&maps.k, k_cam, uint64_t(heads), uint64_t(n_cam), SCA_HEAD_DIM * 2, row, 1, box);
  if (!rc) rc = make_map(&maps.v, v_cam, uint64_t(heads), uint64_t(n_cam), SCA_HEAD_DIM * 2, row, 1, box);
  if (rc) return rc;
  return check_cuda(launch_camera_xattn(maps, a, static_cast<cudaStream_t>(stream)),
                    "camera cross-attention launch");
}

// ---------------------------------------------------------------------------
// work split across the SMs
// ---------------------------------------------------------------------------


static int device_sms(int dev) {
  static std::atomic<int> cached[64] = {};
  if (dev >= 0 && dev < 64) {
    const int c = cached[dev].load(std::memory_order_relaxed);
    if (c) return c;
  }
  int sms = 148;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) sms = 148;
  if (dev >= 0 && dev < 64) cached[dev].store(sms, std::memory_order_relaxed);
  return sms;
}

// Work items are (query-tile pair, head), most expensive pair first, heads
// inner; one CTA runs one item (or one chunk of one). The plan keeps the
// first `n_full` items whole and cuts each of the remaining `n_split` items
// into `chunks` key ranges, so the last wave of SMs is not left half empty. It
// is chosen by simulating greedy dispatch of the CTAs in launch order onto the
// SMs (one CTA per SM), with the pairs' estimated costs plus fixed per-CTA
// and per-split overheads, over a few candidate plans.
static void choose_plan(const sca_metadata* md, int heads, int sms, int forced,
                        int32_t* n_full, int32_t* n_split, int32_t* chunks) {
  const int64_t N = int64_t(md->n_pairs) * heads;
  auto len = [&](int64_t item) {
    return double(md->pair_cost[size_t(md->item_order[size_t(item / heads)])]);
  };
  const double c_cta = 4.0, c_split = 4.0;  // per-CTA start-up; partial store + merge
  auto makespan = [&](int64_t nf, int k) {
    std::priority_queue<double, std::vector<double>, std::greater<double>> q;
    for (int i = 0; i < sms; ++i) q.push(0.0);
    auto run = [&](double cost) {
      const double t = q.top();
      q.pop();
      q.push(t + cost);
    };
    for (int64_t i = 0; i < nf; ++i) run(len(i) + c_cta);
    for (int c = 0; c < k; ++c)
      for (int64_t i = nf; i < N; ++i) run(std::ceil(len(i) / k) + c_cta + c_split);
    double m = 0;
    while (!q.empty()) {
      m = std::max(m, q.top());
      q.pop();
    }
    return m;
  };
  *n_full = int32_t(N);
  *n_split = 0;
  *chunks = 1;
  if (forced == 1 || N == 0) return;
  const int64_t waves = N / sms;
  if (forced >= 2) {
    const int64_t nf = waves >= 1 ? (waves - 1) * sms : 0;
    *n_full = int32_t(nf);
    *n_split = int32_t(N - nf);
    *chunks = forced;
    return;
  }
  double best = makespan(N, 1);
  const int64_t cands[3] = {waves >= 2 ? (waves - 2) * sms : 0, waves >= 1 ? (waves - 1) * sms : 0,
                            waves * sms};
  const int ks[6] = {2, 3, 4, 5, 6, 8};
  for (int64_t nf : cands) {
    if (nf >= N) continue;
    for (int k : ks) {
      const double m = makespan(nf, k);
      if (m < best * 0.995) {  // splitting has to pay for itself
        best = m;
        *n_full = int32_t(nf);
        *n_split = int32_t(N - nf);
        *chunks = k;
      }
    }
  }
}

static void plan_for(const sca_metadata* md, int heads, int dev) {
  const int sms = device_sms(dev);
  const int forced = g_split_override;
  if (md->plan_key[0] == heads && md->plan_key[1] == sms && md->plan_key[2] == forced &&
      md->plan_key[3] == dev)
    return;
  int32_t nf, ns, k;
  choose_plan(md, heads, sms, forced, &nf, &ns, &k);
  md->plan_full = nf;
  md->plan_split = ns;
  md->plan_chunks = k;
  md->plan_ws = k > 1 ? uint64_t(ns) * uint64_t(k) * kPartialSlotBytes : 0;
  md->plan_key[0] = heads;
  md->plan_key[1] = sms;
  md->plan_key[2] = forced;
  md->plan_key[3] = dev;
}

int sca_set_pipeline_timeout_ns(int64_t ns) {
  if (ns < 0 || ns > 10000000000LL)
    return fail(SCA_ERR_INVALID_ARG, "pipeline timeout must be in [0, 10 s]");
  g_pipeline_timeout_ns = (unsigned long long)ns;
  return SCA_OK;
}

int sca_set_split_override(int32_t chunks) {
  if (chunks < 0 || chunks > 64) return fail(SCA_ERR_INVALID_ARG, "split override must be in [0, 64]");
  g_split_override = chunks;
  return SCA_OK;
}

int sca_attn_workspace_bytes(const sca_metadata* md, int32_t heads, uint64_t* bytes) {
  if (!md || !md->built) return fail(SCA_ERR_INVALID_ARG, "metadata not built");
  if (heads < 1 || !bytes) return fail(SCA_ERR_INVALID_ARG, "need heads >= 1 and an output pointer");
  int dev = 0;
  if (int rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice")) return rc;
  plan_for(md, heads, dev);
  *bytes = md->plan_ws;
  return SCA_OK;
}

int sca_attn_int8_scratch_bytes(const sca_metadata* md, int32_t heads, uint64_t* bytes) {
  if (!md || !md->built) return fail(SCA_ERR_INVALID_ARG, "metadata not built");
  if (heads < 1 || !bytes) return fail(SCA_ERR_INVALID_ARG, "need heads >= 1 and an output pointer");
  // bf16 K and V of every cached key, each 256-byte aligned
  *bytes = 2 * align_up(uint64_t(heads) * uint64_t(md->n_cache) * SCA_HEAD_DIM * 2, 256);
  return SCA_OK;
}

int sca_attn_plan(const sca_metadata* md, int32_t heads, int32_t* n_full, int32_t* n_split,
                  int32_t* chunks) {
  if (!md || !md->built) return fail(SCA_ERR_INVALID_ARG, "metadata not built");
  if (heads < 1) return fail(SCA_ERR_INVALID_ARG, "need heads >= 1");
  int dev = 0;
  if (int rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice")) return rc;
  plan_for(md, heads, dev);
  if (n_full) *n_full = md->plan_full;
  if (n_split) *n_split = md->plan_split;
  if (chunks) *chunks = md->plan_chunks;
  return SCA_OK;
}

int sca_attn_plan_for_sms(const sca_metadata* md, int32_t heads, int32_t sms, int32_t* n_full,
                          int32_t* n_split, int32_t* chunks, uint64_t* workspace_bytes) {
  if (!md || !md->built) return fail(SCA_ERR_INVALID_ARG, "metadata not built");
  if (heads < 1 || sms < 1) return fail(SCA_ERR_INVALID_ARG, "need heads >= 1 and sms >= 1");
  int32_t nf, ns, k;
  choose_plan(md, heads, sms, g_split_override, &nf, &ns, &k);
  if (n_full) *n_full = nf;
  if (n_split) *n_split = ns;
  if (chunks) *chunks = k;
  if (workspace_bytes) *workspace_bytes = k > 1 ? uint64_t(ns) * uint64_t(k) * kPartialSlotBytes : 0;
  return SCA_OK;
}

int sca_action_causal_attn_fwd(const sca_kv_cache* cache, const sca_metadata* md, int32_t heads,
                               const void* q, const void* k_cur, const void* v_cur, void* o,
                               float* lse, float softmax_scale, void* workspace,
                               uint64_t workspace_bytes, int32_t* dev_status, void* stream) {
  if (!md || !md->built) return fail(SCA_ERR_INVALID_ARG, "metadata not built");
  if (!md->uploaded) return fail(SCA_ERR_INVALID_ARG, "metadata not uploaded");
  if (heads < 1) return fail(SCA_ERR_INVALID_ARG, "heads must be >= 1");
  if (!q || !k_cur || !v_cur || !o) return fail(SCA_ERR_INVALID_ARG, "null q, k_cur, v_cur or o");
  if (!aligned16(q) || !aligned16(k_cur) || !aligned16(v_cur) || !aligned16(o) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return fail(SCA_ERR_MISALIGNED, "q, k_cur, v_cur, o must be 16-byte aligned (lse 4-byte)");
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(SCA_ERR_MISALIGNED, "workspace must be 256-byte aligned");
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale))
    return fail(SCA_ERR_INVALID_ARG, "softmax_scale must be positive and finite");
  if (md->n_cached > 0) {
    if (!cache) return fail(SCA_ERR_MISMATCH, "metadata has cached segments but no cache was given");
    if (cache->heads != heads) return fail(SCA_ERR_MISMATCH, "cache has %d heads, call has %d", cache->heads, heads);
    if (cache->segs.size() != size_t(md->n_cached))
      return fail(SCA_ERR_MISMATCH, "cache holds %zu segments, metadata expects %d",
                  cache->segs.size(), md->n_cached);
    for (int i = 0; i < md->n_cached; ++i)
      if (!cache->segs[size_t(i)].same(md->segs[size_t(i)]))
        return fail(SCA_ERR_MISMATCH, "cached segment %d differs from the metadata's layout", i);
  }
  int dev = 0;
  if (int rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice")) return rc;
  if (dev != md->device) return fail(SCA_ERR_MISMATCH, "metadata was uploaded to another device");
  if (int64_t(md->n_pairs) * heads * 64 > INT32_MAX) return fail(SCA_ERR_UNSUPPORTED, "grid too large");

  const uint64_t row = uint64_t(heads) * SCA_HEAD_DIM * 2;  // bytes per token, token-major
  AttnMaps maps;
  memset(&maps, 0, sizeof(maps));
  int rc = make_map(&maps.q, q, uint64_t(heads), uint64_t(md->n_q), SCA_HEAD_DIM * 2, row, 1, SCA_TILE);
  if (!rc) rc = make_map(&maps.k_cur, k_cur, uint64_t(heads), uint64_t(md->n_q), SCA_HEAD_DIM * 2, row, 1, SCA_TILE);
  if (!rc) rc = make_map(&maps.v_cur, v_cur, uint64_t(heads), uint64_t(md->n_q), SCA_HEAD_DIM * 2, row, 1, SCA_TILE);
  bool int8_cache = md->n_cache > 0 && cache->int8;
  // An INT8 cache with room for a bf16 copy of it after the split scratch:
  // dequantise once here and run the bf16 kernel on the copy (the same
  // values reach the products as in the kernel that dequantises tile by tile).
  plan_for(md, heads, dev);
  uint64_t scratch = 0;
  if (int8_cache) sca_attn_int8_scratch_bytes(md, heads, &scratch);
  const uint64_t split_ws = align_up(md->plan_ws, 256);
  const bool via_scratch = int8_cache && workspace && workspace_bytes >= split_ws + scratch;
  if (!rc && via_scratch) {
    uint8_t* base = static_cast<uint8_t*>(workspace) + split_ws;
    DequantArgs dq{};
    dq.k_codes = cache->k;
    dq.v_codes = cache->v;
    dq.k_scale = cache->k_scale;
    dq.v_scale = cache->v_scale;
    dq.k_out = base;
    dq.v_out = base + scratch / 2;
    dq.n = md->n_cache;
    dq.capacity = cache->capacity;
    dq.heads = heads;
    if (int rc2 = check_cuda(launch_dequant(dq, static_cast<cudaStream_t>(stream)), "dequant launch"))
      return rc2;
    const uint64_t hstride = uint64_t(md->n_cache) * SCA_HEAD_DIM * 2;
    rc = make_map(&maps.k_cache, dq.k_out, uint64_t(md->n_cache), uint64_t(heads), SCA_HEAD_DIM * 2,
                  hstride, SCA_TILE, 1);
    if (!rc) rc = make_map(&maps.v_cache, dq.v_out, uint64_t(md->n_cache), uint64_t(heads),
                           SCA_HEAD_DIM * 2, hstride, SCA_TILE, 1);
    int8_cache = false;  // the bf16 kernel reads the copy
  } else if (!rc && int8_cache) {
    const uint64_t n = uint64_t(md->n_cache), cap = uint64_t(cache->capacity);
    rc = make_code_map(&maps.k_cache, cache->k, n, uint64_t(heads), cap);
    if (!rc) rc = make_code_map(&maps.v_cache, cache->v, n, uint64_t(heads), cap);
    if (!rc) rc = make_scale_map(&maps.k_scale, cache->k_scale, n, uint64_t(heads), cap);
    if (!rc) rc = make_scale_map(&maps.v_scale, cache->v_scale, n, uint64_t(heads), cap);
  } else if (!rc && md->n_cache > 0) {
    const uint64_t hstride = uint64_t(cache->capacity) * SCA_HEAD_DIM * 2;
    rc = make_map(&maps.k_cache, cache->k, uint64_t(md->n_cache), uint64_t(heads), SCA_HEAD_DIM * 2,
                  hstride, SCA_TILE, 1);
    if (!rc) rc = make_map(&maps.v_cache, cache->v, uint64_t(md->n_cache), uint64_t(heads),
                           SCA_HEAD_DIM * 2, hstride, SCA_TILE, 1);
  }
  if (rc) return rc;

  const uint8_t* d = static_cast<const uint8_t*>(md->dev);
  AttnArgs a{};
  a.qdesc = reinterpret_cast<const uint2*>(d + md->off_qdesc);
  a.item_order = reinterpret_cast<const int32_t*>(d + md->off_order);
  a.pair_ptr = reinterpret_cast<const int32_t*>(d + md->off_ptr);
  a.pair_list = reinterpret_cast<const uint32_t*>(d + md->off_list);
  a.run_ptr = reinterpret_cast<const int32_t*>(d + md->off_run_ptr);
  a.runs = reinterpret_cast<const uint2*>(d + md->off_runs);
  a.o = o;
  a.lse = lse;
  a.status = dev_status;
  a.n_q = int32_t(md->n_q);
  a.n_cache = int32_t(md->n_cache);
  a.n_cache_tiles = md->n_cache_tiles;
  a.heads = heads;
  a.n_pairs = md->n_pairs;
  a.history = md->history;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.timeout_ns = g_pipeline_timeout_ns;
  const bool split = md->plan_chunks > 1 && workspace && workspace_bytes >= md->plan_ws;
  a.n_full = split ? md->plan_full : md->n_pairs * heads;
  a.n_split = split ? md->plan_split : 0;
  a.chunks = split ? md->plan_chunks : 1;
  if (split) {
    const uint64_t slots = uint64_t(a.n_split) * uint64_t(a.chunks);
    a.part_o = static_cast<float*>(workspace);
    a.part_ml = reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) + slots * 256 * 128 * 4);
  }
  if (int rc2 = check_cuda(launch_attention(maps, a, int8_cache, static_cast<cudaStream_t>(stream)),
                           "attention launch"))
    return rc2;
  if (split)
    return check_cuda(launch_merge(a, static_cast<cudaStream_t>(stream)), "merge launch");
  return SCA_OK;
}

int sca_attn_bwd_workspace_bytes(const sca_metadata* md, int32_t heads, uint64_t* bytes) {
  if (!md || !md->built) return fail(SCA_ERR_INVALID_ARG, "metadata not built");
  if (heads < 1 || !bytes) return fail(SCA_ERR_INVALID_ARG, "need heads >= 1 and an output");
  *bytes = 2ull * uint64_t(heads) * uint64_t(md->n_q_tiles) * SCA_TILE * 4;
  return SCA_OK;
}

int sca_action_causal_attn_bwd(const sca_metadata* md, int32_t heads, const void* q, const void* k,
                               const void* v, const void* o, const float* lse, const void* d_o,
                               void* dq, void* dk, void* dv, float softmax_scale, void* workspace,
                               uint64_t workspace_bytes, int32_t* dev_status, void* stream) {
  if (!md || !md->built) return fail(SCA_ERR_INVALID_ARG, "metadata not built");
  if (!md->uploaded) return fail(SCA_ERR_INVALID_ARG, "metadata not uploaded");
  if (md->n_cached > 0)
    return fail(SCA_ERR_UNSUPPORTED, "the backward pass takes layouts without cached segments");
  if (heads < 1) return fail(SCA_ERR_INVALID_ARG, "heads must be >= 1");
  if (!q || !k || !v || !o || !lse || !d_o || !dq || !dk || !dv)
    return fail(SCA_ERR_INVALID_ARG, "null q, k, v, o, lse, d_o, dq, dk or dv");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(d_o) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(SCA_ERR_MISALIGNED, "tensors must be 16-byte aligned (lse 4-byte)");
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale))
    return fail(SCA_ERR_INVALID_ARG, "softmax_scale must be positive and finite");
  uint64_t need = 0;
  sca_attn_bwd_workspace_bytes(md, heads, &need);
  if (!workspace || workspace_bytes < need)
    return fail(SCA_ERR_CAPACITY, "the backward pass needs a workspace of %llu bytes",
                (unsigned long long)need);
  if (reinterpret_cast<uintptr_t>(workspace) & 255u)
    return fail(SCA_ERR_MISALIGNED, "workspace must be 256-byte aligned");
  int dev = 0;
  if (int rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice")) return rc;
  if (dev != md->device) return fail(SCA_ERR_MISMATCH, "metadata was uploaded to another device");
  if (int64_t(md->n_pairs) * 2 * heads > INT32_MAX) return fail(SCA_ERR_UNSUPPORTED, "grid too large");

  const uint64_t n = uint64_t(md->n_q), n_pad = uint64_t(md->n_q_tiles) * SCA_TILE;
  const uint64_t row = uint64_t(heads) * SCA_HEAD_DIM * 2;
  BwdMaps maps;
  memset(&maps, 0, sizeof(maps));
  int rc = make_map(&maps.q, q, uint64_t(heads), n, SCA_HEAD_DIM * 2, row, 1, SCA_TILE);
  if (!rc) rc = make_map(&maps.k, k, uint64_t(heads), n, SCA_HEAD_DIM * 2, row, 1, SCA_TILE);
  if (!rc) rc = make_map(&maps.v, v, uint64_t(heads), n, SCA_HEAD_DIM * 2, row, 1, SCA_TILE);
  if (!rc) rc = make_map(&maps.d_o, d_o, uint64_t(heads), n, SCA_HEAD_DIM * 2, row, 1, SCA_TILE);
  if (!rc) rc = make_scale_map(&maps.dl, static_cast<const float*>(workspace), n_pad,
                               2 * uint64_t(heads), n_pad);
  if (rc) return rc;

  const uint8_t* d = static_cast<const uint8_t*>(md->dev);
  BwdArgs a{};
  a.item_order = reinterpret_cast<const int32_t*>(d + md->off_order);
  a.pair_ptr = reinterpret_cast<const int32_t*>(d + md->off_ptr);
  a.pair_list = reinterpret_cast<const uint32_t*>(d + md->off_list);
  a.run_ptr = reinterpret_cast<const int32_t*>(d + md->off_run_ptr);
  a.runs = reinterpret_cast<const uint2*>(d + md->off_runs);
  a.qdesc = reinterpret_cast<const uint2*>(d + md->off_qdesc);
  a.kt_order = reinterpret_cast<const int32_t*>(d + md->off_kt_order);
  a.kt_ptr = reinterpret_cast<const int32_t*>(d + md->off_kt_ptr);
  a.kt_list = reinterpret_cast<const uint32_t*>(d + md->off_kt_list);
  a.qrun_ptr = reinterpret_cast<const int32_t*>(d + md->off_qrun_ptr);
  a.qruns = reinterpret_cast<const uint4*>(d + md->off_qruns);
  a.kdesc = reinterpret_cast<const uint32_t*>(d + md->off_kdesc);
  a.o = o;
  a.d_o = d_o;
  a.lse = lse;
  a.dl = static_cast<float*>(workspace);
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.status = dev_status;
  a.n = int32_t(n);
  a.n_pad = int32_t(n_pad);
  a.heads = heads;
  a.n_q_tiles = md->n_q_tiles;
  a.n_pairs = md->n_pairs;
  a.history = md->history;
  a.scale = softmax_scale;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.timeout_ns = g_pipeline_timeout_ns;
  return check_cuda(launch_backward(maps, a, static_cast<cudaStream_t>(stream)), "backward launch");
}

int sca_read_device_status(const int32_t* dev_status, void* stream) {
  if (!dev_status) return fail(SCA_ERR_INVALID_ARG, "null status word");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (int rc = check_cuda(cudaMemcpyAsync(&v, dev_status, sizeof(v), cudaMemcpyDeviceToHost, st),
                          "cudaMemcpyAsync(status)"))
    return rc;
  if (int rc = check_cuda(cudaStreamSynchronize(st), "cudaStreamSynchronize")) return rc;
  switch (v) {
    case SCA_OK: return SCA_OK;
    case SCA_ERR_DEVICE_TIMEOUT:
      return fail(v, "a kernel's bounded wait ran out (device status %d)", v);
    case SCA_ERR_MISALIGNED:
      return fail(v, "a kernel's shared-memory window was misaligned (device status %d)", v);
    default:
      return fail(v < 0 ? v : SCA_ERR_CUDA, "device status word holds %d", v);
  }
}

int sca_debug_bounded_wait(int32_t* dev_status, int64_t timeout_ns, void* stream) {
  if (!dev_status) return fail(SCA_ERR_INVALID_ARG, "null status");
  if (timeout_ns < 0 || timeout_ns > 10000000000LL)
    return fail(SCA_ERR_INVALID_ARG, "timeout must be in [0, 10 s]");
  return check_cuda(launch_bounded_wait(dev_status, (unsigned long long)timeout_ns,
                                        static_cast<cudaStream_t>(stream)),
                    "bounded-wait launch");
}

}  // extern "C"
