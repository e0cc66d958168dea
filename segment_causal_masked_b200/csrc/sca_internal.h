// Internal declarations shared by the host runtime (sca_host.cpp) and the
// device kernels (sca_kernels.cu). Not part of the ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "sca.h"

namespace sca {

// Validated copy of one segment's layout.
struct SegLayout {
  int32_t F = 0, G = 0, h = 0, n_act = 0;
  int32_t len[SCA_MAX_ACTIONS] = {};
  int32_t beg[SCA_MAX_ACTIONS] = {};
  int32_t end[SCA_MAX_ACTIONS] = {};
  int64_t n_video() const { return int64_t(F) * G; }
  int64_t n_tokens() const {
    int64_t n = n_video() + h;
    for (int a = 0; a < n_act; ++a) n += len[a];
    return n;
  }
  // bit a set when frame f lies in action a's window
  uint32_t frame_mask(int f) const {
    uint32_t m = 0;
    for (int a = 0; a < n_act; ++a)
      if (beg[a] <= f && f < end[a]) m |= 1u << a;
    return m;
  }
  uint32_t all_actions() const {
    return n_act >= 32 ? 0xFFFFFFFFu : ((1u << n_act) - 1u);
  }
  bool same(const SegLayout& o) const;
};

// Sets the thread's message and returns `code`.
int fail(int code, const char* fmt, ...);
int check_cuda(cudaError_t e, const char* what);
int read_segment(const sca_segment* s, SegLayout* out);
// The calling thread's key-split override (sca_set_split_override).
int split_override();

// Descriptor word of token `t` (0-based inside the segment).
uint32_t key_descriptor(const SegLayout& s, uint32_t seg_index, int64_t t);

// ---------------------------------------------------------------------------
// device-side views
// ---------------------------------------------------------------------------

// Pair work list entry: bits 0..23 key tile, bits 24..25 class for the
// first query tile of the pair, bits 26..27 for the second.
constexpr uint32_t kPairTileMask = 0xFFFFFFu;

struct AttnArgs {
  // metadata (device)
  const uint2* qdesc;          // [n_pairs * 256]
  const int32_t* item_order;   // [n_pairs] longest list first
  const int32_t* pair_ptr;     // [n_pairs + 1]
  const uint32_t* pair_list;   // [pair_ptr[n_pairs]]
  const int32_t* run_ptr;      // [n_kv_tiles + 1] runs of each key tile
  const uint2* runs;           // {first column | count << 8, key descriptor}
  // outputs
  void* o;                     // bf16 [n_q][heads][128]
  float* lse;                  // [heads][n_q] or null
  int32_t* status;             // device status word or null
  // split-KV tail: CTAs [0, n_full) run whole items; the next
  // n_split * chunks CTAs run chunk k of item n_full + si (chunk-major) and
  // write fp32 partials (unnormalised O, running max and sum, log2 domain)
  // to slot si * chunks + k
  float* part_o;               // [slots][256][128]
  float2* part_ml;             // [slots][256]
  int32_t n_full;
  int32_t n_split;
  int32_t chunks;
  // sizes
  int32_t n_q;
  int32_t n_cache;             // cache keys
  int32_t n_cache_tiles;
  int32_t heads;
  int32_t n_pairs;
  int32_t history;             // earlier segments a query may see (65535: all)
  float scale_log2;            // softmax_scale * log2(e)
  unsigned long long timeout_ns;
};

// For an INT8 cache, k_cache / v_cache cover the int8 codes (rows of 128
// bytes) and k_scale / v_scale the per-row fp32 scales.
struct AttnMaps {
  CUtensorMap q, k_cur, v_cur, k_cache, v_cache, k_scale, v_scale;
};

cudaError_t launch_attention(const AttnMaps& maps, const AttnArgs& args, bool int8_cache,
                             cudaStream_t stream);
cudaError_t launch_merge(const AttnArgs& args, cudaStream_t stream);

// bytes of one partial slot: O [256][128] fp32 + (m, l) [256]
constexpr uint64_t kPartialSlotBytes = 256ull * 128 * 4 + 256ull * 8;

struct AppendArgs {
  const void* k;
  const void* v;
  void* k_cache;
  void* v_cache;
  float* k_scale;       // INT8 cache: per-row scales (k_cache / v_cache hold codes)
  float* v_scale;
  int32_t int8;         // 0: bf16 cache, 1: INT8 cache
  uint32_t* desc;
  int64_t length;       // first row written
  int64_t capacity;
  int32_t n;            // tokens of the segment
  int32_t heads;
  uint32_t seg_index;
  int32_t n_video;
  int32_t head_len;
  int32_t n_act;
  int32_t tail_start[SCA_MAX_ACTIONS + 1];  // offsets of the tails after the head
};

cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream);

// INT8 cache rows [0, n) of every head -> bf16 [heads][n][128].
struct DequantArgs {
  const void* k_codes;
  const void* v_codes;
  const float* k_scale;
  const float* v_scale;
  void* k_out;
  void* v_out;
  int64_t n;
  int64_t capacity;
  int32_t heads;
};
cudaError_t launch_dequant(const DequantArgs& a, cudaStream_t stream);

// Attention backward (layouts without cached segments: keys = queries = the
// n current tokens). Work-list views of the metadata, the workspace and the
// tensors of one call.
struct BwdArgs {
  const int32_t* item_order;   // query-tile pairs, most expensive first
  const int32_t* pair_ptr;     // [n_pairs + 1]
  const uint32_t* pair_list;   // key tile | class of tile 0 << 24 | class of tile 1 << 26
  const int32_t* run_ptr;      // key runs per key tile
  const uint2* runs;
  const uint2* qdesc;          // [n_pairs * 256] query descriptors
  const int32_t* kt_order;     // key tiles, longest list first
  const int32_t* kt_ptr;       // [n_kv_tiles + 1]
  const uint32_t* kt_list;     // query tile | class << 24 (non-EMPTY only, ascending)
  const int32_t* qrun_ptr;     // [n_q_tiles + 1] query runs per query tile
  const uint4* qruns;          // {first | count << 8, query word 0, query word 1, 0}
  const uint32_t* kdesc;       // [n_q_tiles * 128] key descriptor per token (0 past n)
  const void* o;               // bf16 [n][heads][128]
  const void* d_o;
  const float* lse;            // [heads][n], natural log
  float* dl;                   // workspace [2][heads][n_pad]: D, then LSE * log2(e)
  void* dq;                    // bf16 [n][heads][128]
  void* dk;
  void* dv;
  int32_t* status;
  int32_t n;
  int32_t n_pad;               // round_up(n, 128)
  int32_t heads;
  int32_t n_q_tiles;
  int32_t n_pairs;
  int32_t history;
  float scale;
  float scale_log2;
  unsigned long long timeout_ns;
};

struct BwdMaps {
  CUtensorMap q, k, v, d_o;    // token-major bf16, box (64, 1, 128)
  CUtensorMap dl;              // workspace rows, box (128, 1)
};

cudaError_t launch_backward(const BwdMaps& maps, const BwdArgs& args, cudaStream_t stream);
cudaError_t launch_bounded_wait(int32_t* status, unsigned long long timeout_ns,
                                cudaStream_t stream);

size_t attention_smem_bytes(bool int8_cache);

}  // namespace sca

// ---------------------------------------------------------------------------
// opaque handles
// ---------------------------------------------------------------------------

struct sca_metadata {
  bool built = false;
  int32_t n_cached = 0, n_current = 0, policy = 0;
  int32_t history = 65535;            // window over earlier segments (65535: all)
  int64_t n_dropped = 0;              // video blocks dropped by keep_blocks
  std::vector<sca::SegLayout> segs;   // cached then current
  int64_t n_cache = 0;                // cached keys
  int64_t n_q = 0;                    // queries = current keys
  int64_t unmasked_pairs = 0;
  int32_t n_q_tiles = 0, n_cache_tiles = 0, n_kv_tiles = 0, n_pairs = 0;
  int64_t n_full = 0, n_partial = 0;
  // host outputs
  std::vector<uint32_t> key_desc_cur;  // [n_q]
  std::vector<uint32_t> query_desc;    // [2 n_q]
  std::vector<int32_t> row_ptr;        // [n_q_tiles + 1]
  std::vector<int32_t> kv_tile;        // [nnz]
  std::vector<uint8_t> flag;           // [nnz]
  std::vector<int32_t> pair_ptr;       // [n_pairs + 1]
  std::vector<uint32_t> pair_list;
  std::vector<int32_t> item_order;     // [n_pairs], most expensive first
  std::vector<float> pair_cost;        // [n_pairs] estimated cost (query-tile x key-tile units)
  std::vector<int32_t> run_ptr;        // [n_kv_tiles + 1]
  std::vector<uint32_t> runs;          // pairs of words: first | count << 8, descriptor
  // backward (layouts without a cache only)
  std::vector<int32_t> kt_ptr;         // [n_kv_tiles + 1]
  std::vector<uint32_t> kt_list;       // query tile | class << 24
  std::vector<int32_t> kt_order;       // key tiles, most expensive first
  std::vector<int32_t> qrun_ptr;       // [n_q_tiles + 1]
  std::vector<uint32_t> qruns;         // 4 words: first | count << 8, query words 0 and 1, 0
  std::vector<uint32_t> kdesc_pad;     // [n_q_tiles * 128]
  // device copy
  bool uploaded = false;
  int device = -1;
  void* dev = nullptr;
  size_t dev_bytes = 0;
  void* pinned = nullptr;
  size_t pinned_bytes = 0;
  cudaEvent_t upload_done = nullptr;
  size_t off_qdesc = 0, off_order = 0, off_ptr = 0, off_list = 0;
  size_t off_run_ptr = 0, off_runs = 0;
  size_t off_kt_ptr = 0, off_kt_list = 0, off_kt_order = 0, off_qrun_ptr = 0, off_qruns = 0,
         off_kdesc = 0;
  // last split plan (heads, SMs, workspace, override) -> plan
  mutable int32_t plan_key[4] = {-1, -1, -1, -1};
  mutable uint64_t plan_ws = 0;
  mutable int32_t plan_full = 0, plan_split = 0, plan_chunks = 1;
};

struct sca_kv_cache {
  int32_t heads = 0;
  int64_t capacity = 0;
  bool int8 = false;          // codes + scales instead of bf16 rows
  void* k = nullptr;          // bf16 rows, or int8 codes
  void* v = nullptr;
  float* k_scale = nullptr;   // INT8 only
  float* v_scale = nullptr;
  uint32_t* desc = nullptr;
  int64_t length = 0;
  std::vector<sca::SegLayout> segs;
  std::vector<int64_t> seg_start;
};
