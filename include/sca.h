/*
 * sca.h - C ABI of libsca: action-aware causal joint attention over a growing
 * KV cache, for NVIDIA B200 (sm_100a).
 *
 * The operation (Hy-Nomas pages):
 *   - attention is bidirectional inside a segment and causal across segments
 *     (picx.dev summary, Model Architecture, "Segment-wise Causal Attention");
 *   - a segment's text is a descriptive head plus action tails a_0..a_n, each
 *     with a window of latent frames; a query inside an action's window sees
 *     that tail and the head; heads stay visible to later segments, tails
 *     never leave their own segment (same page, "Action-Aware Causal
 *     Attention (Figure 6b)"; onedev.kr review, "무엇과 다른가");
 *   - after a segment is generated its K/V joins a permanent cache that later
 *     segments attend to (gpts24.com, "One World, Generated Segment by
 *     Segment");
 *   - A, the number of unmasked query-key pairs, is the A_i of Eq. 6 (picx.dev
 *     summary, Training Infrastructure; xyznot.com, "Dağıtık Paketleme FLOP
 *     Tahmini").
 *
 * Conventions shared by every call:
 *   - Return value 0 on success, a negative SCA_ERR_* code on failure; the
 *     calling thread's message is then available from sca_last_error().
 *     A call that fails validation has no effect (nothing is written, nothing
 *     is enqueued). No C++ exception crosses this ABI.
 *   - Device pointers are plain CUDA global-memory addresses owned by the
 *     caller (e.g. PyTorch tensors). The library owns only its opaque handles.
 *   - Work is enqueued on the caller's stream (cudaStream_t passed as void*;
 *     NULL is the legacy default stream) and runs asynchronously; device-side
 *     failures (a bounded wait that timed out) are reported through the
 *     optional device status word.
 *   - Tensors are bf16 with head dimension d = 128. Token-major tensors are
 *     [tokens][heads][128] contiguous; the cache is head-major
 *     [heads][capacity][128] contiguous.
 *   - Every device pointer must be 16-byte aligned (TMA and 16-byte vector
 *     access); otherwise SCA_ERR_MISALIGNED.
 *   - Threads: different handles may be used from different host threads at
 *     once. One handle (a metadata or a cache) must not be used by two
 *     threads at the same time, even through calls that take it as const
 *     (the attention call caches its work split in the metadata handle).
 */
#ifndef SCA_H_
#define SCA_H_

#include <stdint.h>

#if defined(__GNUC__)
#define SCA_API __attribute__((visibility("default")))
#else
#define SCA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define SCA_HEAD_DIM 128
#define SCA_TILE 128
#define SCA_MAX_ACTIONS 32
#define SCA_MAX_SEGMENTS 65535

enum {
  SCA_OK = 0,
  SCA_ERR_INVALID_ARG = -1,   /* bad layout, size or pointer */
  SCA_ERR_UNSUPPORTED = -2,   /* head_dim != 128, too many segments/tiles */
  SCA_ERR_MISALIGNED = -3,    /* a device pointer is not 16-byte aligned */
  SCA_ERR_CAPACITY = -4,      /* the cache cannot hold the appended segment */
  SCA_ERR_CUDA = -5,          /* a CUDA runtime/driver call failed */
  SCA_ERR_DEVICE_TIMEOUT = -6,/* a kernel's bounded wait ran out (device status) */
  SCA_ERR_MISMATCH = -7       /* metadata does not describe this cache */
};

/* Text-query convention. The pages state what video queries see; for text
 * queries they are silent.
 *   SCA_TEXTQ_OWN_TAIL (default): a head query sees its own segment's video
 *     and head; a query in tail a also sees tail a; no earlier segment.
 *   SCA_TEXTQ_FULL_SEGMENT: a text query sees its whole own segment and, like
 *     a video query, the video and heads of earlier segments. */
enum { SCA_TEXTQ_OWN_TAIL = 0, SCA_TEXTQ_FULL_SEGMENT = 1 };

/* Tile classes of the schedule. */
enum { SCA_TILE_EMPTY = 0, SCA_TILE_PARTIAL = 1, SCA_TILE_FULL = 2 };

/* Key descriptor word (one per key; the cache's descriptor array and the
 * current segments' keys):
 *   bits 0..15 segment index (cache segments first, in time order),
 *   bit 16 action tail, bit 17 alive (visible to later segments: video and
 *   head), bit 18 descriptive head, bits 24..29 action index of a tail.
 * Query descriptor: two words per query,
 *   word 0: bits 0..15 segment index, bit 16 sees earlier segments,
 *           bit 17 valid query;
 *   word 1: bit a set when the query sees tail a of its own segment. */
#define SCA_DESC_SEG_MASK 0xFFFFu
#define SCA_DESC_TAIL (1u << 16)
#define SCA_DESC_ALIVE (1u << 17)
#define SCA_DESC_HEAD (1u << 18)
#define SCA_DESC_ACTION_SHIFT 24
#define SCA_QDESC_SEES_PAST (1u << 16)
#define SCA_QDESC_VALID (1u << 17)

/* One segment's layout. Token order inside a segment: video frame by frame
 * (num_frames * tokens_per_frame tokens), then the head (head_len tokens),
 * then tail 0, tail 1, ... (action_len[a] tokens each). Action a's window is
 * the half-open latent-frame range [action_begin[a], action_end[a]) local to
 * the segment. Requirements: num_frames >= 1, tokens_per_frame >= 1,
 * head_len >= 0, 0 <= num_actions <= 32, action_len[a] >= 1,
 * 0 <= begin < end <= num_frames. The arrays are read during the call only. */
typedef struct sca_segment {
  int32_t num_frames;
  int32_t tokens_per_frame;
  int32_t head_len;
  int32_t num_actions;
  const int32_t* action_len;
  const int32_t* action_begin;
  const int32_t* action_end;
} sca_segment;

typedef struct sca_metadata sca_metadata; /* mask metadata + tile schedule */
typedef struct sca_kv_cache sca_kv_cache; /* growing KV cache */

/* ---------------------------------------------------------------------------
 * Metadata: per-token descriptors and the block-sparse tile schedule.
 *
 * Keys are the tokens of `cached` (in time order) followed by those of
 * `current`; queries are the tokens of `current`. With n_cached = 0 and
 * several current segments this is a packed training-shaped call.
 *
 * Tiles: query tile i = queries [128 i, 128 i + 128). Key tiles are 128
 * consecutive keys of one source: cache tiles t < nC = ceil(n_cache/128)
 * cover cache keys [128 t, 128 t + 128); tile nC + u covers current keys
 * [128 u, 128 u + 128). A (query tile, key tile) pair is FULL when all
 * 128x128 positions exist and are visible, EMPTY when no existing position is
 * visible, PARTIAL otherwise. The schedule lists each query tile's non-EMPTY
 * key tiles in ascending order (CSR).
 * ------------------------------------------------------------------------- */

/* Create an empty handle. */
SCA_API int sca_metadata_create(sca_metadata** out);

/* Build descriptors, schedule and A on the host (no GPU needed). Replaces the
 * handle's previous contents. Requires n_current >= 1 and
 * n_cached + n_current <= 65535. SCA_ERR_INVALID_ARG on a bad layout. */
SCA_API int sca_build_segment_mask_metadata(sca_metadata* md,
                                    const sca_segment* cached, int32_t n_cached,
                                    const sca_segment* current, int32_t n_current,
                                    int32_t textq_policy);

/* Options of the mask (all optional; zero-initialise and set what you need).
 * The inference path of the Hy-Nomas report names sliding-window attention
 * and sparse attention that keeps a quarter of the video blocks (picx.dev
 * summary, "Inference") without their rules; this library reads them as:
 *   history_segments W >= 0: a query of segment s sees earlier segments
 *     s-W .. s-1 only (its own segment as always); -1 (or any negative) keeps
 *     the whole history. 0 is a valid window (no earlier segment).
 *   keep_blocks: NULL keeps everything; else n_q_tiles * n_kv_tiles bytes,
 *     row-major [query tile][key tile] (tiles as in the schedule; get the
 *     counts from a build without it): a 0 entry drops, for that query tile,
 *     the whole key tile when it holds video tokens only ("a video block").
 *     Key tiles with any text key are kept whatever the entry. Dropped
 *     blocks leave the schedule and the unmasked-pair count. */
typedef struct sca_mask_options {
  int32_t textq_policy;
  int32_t history_segments;
  const uint8_t* keep_blocks;
  int64_t keep_blocks_len;
} sca_mask_options;

/* sca_build_segment_mask_metadata with options (opt may be NULL: defaults,
 * i.e. SCA_TEXTQ_OWN_TAIL, whole history, every block).
 * SCA_ERR_INVALID_ARG if keep_blocks_len does not match the layout's tiles. */
SCA_API int sca_build_segment_mask_metadata_ex(sca_metadata* md,
                                               const sca_segment* cached, int32_t n_cached,
                                               const sca_segment* current, int32_t n_current,
                                               const sca_mask_options* opt);

/* Sizes and totals of the last build. Any output pointer may be NULL.
 *   unmasked_pairs: A (pairs whose mask entry is not -inf), per head;
 *   n_queries / n_cache_keys: token counts; n_q_tiles, n_kv_tiles: tiles;
 *   nnz / n_full / n_partial: entries of the schedule and their classes. */
SCA_API int sca_metadata_get_counts(const sca_metadata* md, int64_t* unmasked_pairs,
                            int64_t* n_queries, int64_t* n_cache_keys,
                            int32_t* n_q_tiles, int32_t* n_kv_tiles, int64_t* nnz,
                            int64_t* n_full, int64_t* n_partial);

/* Host views of the schedule (CSR: row_ptr[n_q_tiles+1], kv_tile[nnz],
 * flag[nnz] with SCA_TILE_PARTIAL/FULL) and of the descriptors of the
 * current keys (key_desc[n_queries]) and queries (query_desc[2 n_queries]).
 * The pointers stay valid until the next build or destroy. */
SCA_API int sca_metadata_get_schedule(const sca_metadata* md, const int32_t** row_ptr,
                              const int32_t** kv_tile, const uint8_t** flag);
SCA_API int sca_metadata_get_descriptors(const sca_metadata* md, const uint32_t** key_desc,
                                 const uint32_t** query_desc);

/* Copy the device-side part (descriptors and the kernel's work list) to the
 * GPU, on `stream`, through a pinned staging buffer the handle owns. Device
 * and staging buffers grow on demand (the call that grows them allocates and
 * may synchronize); a rebuilt handle of the same size reuses them. The
 * staging buffer is only rewritten after the previous upload has completed. */
SCA_API int sca_metadata_upload(sca_metadata* md, void* stream);

SCA_API void sca_metadata_destroy(sca_metadata* md);

/* ---------------------------------------------------------------------------
 * KV cache. The caller allocates, the cache object only records them:
 *   k_buf, v_buf: bf16 [heads][capacity][128] (head-major);
 *   desc_buf:     uint32 [round_up(capacity, 128)] key descriptor words.
 * ------------------------------------------------------------------------- */
SCA_API int sca_kv_cache_create(sca_kv_cache** out, int32_t heads, int32_t head_dim,
                        int64_t capacity, void* k_buf, void* v_buf, void* desc_buf);

/* INT8 KV cache (Hy-Nomas summary on picx.dev, "Inference": the cache may be
 * quantised to INT8 for single-GPU inference; the pages give no scheme).
 * Each 128-value row of K or V (one token, one head) is stored as int8 codes
 * with one fp32 scale:
 *     scale = max_d |x_d| / 127,   code_d = round_half_even(x_d / scale)
 * in fp32 from the bf16 values (a zero row: scale 0, codes 0), clamped to
 * [-127, 127]; the cached value is code * scale. Caller-owned buffers:
 *   k_codes, v_codes: uint8 [heads][capacity][128], each code stored
 *                     offset-binary as code + 128 (1 ... 255);
 *   k_scale, v_scale: fp32 [heads][capacity];
 *   desc_buf:         uint32 [round_up(capacity, 128)] as above.
 * capacity must be a multiple of 4 (the scale rows are read with 16-byte
 * aligned tensor copies): SCA_ERR_INVALID_ARG otherwise. The buffers must be
 * 16-byte aligned (SCA_ERR_MISALIGNED). sca_kv_cache_append quantises while
 * it copies (bit for bit the rule above); attention reads the codes and
 * scales and dequantises tile by tile in shared memory, with the scaled
 * value rounded to bf16 before the products. Appending and truncating work
 * as for a bf16 cache. */
SCA_API int sca_kv_cache_create_int8(sca_kv_cache** out, int32_t heads, int32_t head_dim,
                                     int64_t capacity, void* k_codes, void* v_codes,
                                     float* k_scale, float* v_scale, void* desc_buf);

/* Append one segment: copy its keys and values k, v (bf16 token-major
 * [n][heads][128], n = the segment's token count) into cache rows
 * [length, length + n) of every head with 16-byte coalesced stores, write its
 * key descriptors with the tails marked dead (alive bit clear), and advance
 * the length. SCA_ERR_CAPACITY if length + n > capacity. */
SCA_API int sca_kv_cache_append(sca_kv_cache* cache, const sca_segment* segment,
                        const void* k, const void* v, void* stream);

/* Forget every segment after the first n_segments (host-side; the buffers
 * keep their bytes). */
SCA_API int sca_kv_cache_truncate(sca_kv_cache* cache, int32_t n_segments);

/* Length in keys and number of segments. Either pointer may be NULL. */
SCA_API int sca_kv_cache_get(const sca_kv_cache* cache, int64_t* length, int32_t* n_segments);

SCA_API void sca_kv_cache_destroy(sca_kv_cache* cache);

/* ---------------------------------------------------------------------------
 * Attention forward.
 *
 * For every head h and query i (a token of the metadata's current segments):
 *   s_ik = softmax_scale * <q_ih, k_kh> for the keys k that i may see,
 *   o_ih = sum_k softmax_k(s_i) v_kh,  lse[h][i] = log sum_k exp(s_ik),
 * keys being the cache's keys followed by k_cur. bf16 inputs and outputs,
 * fp32 accumulation. Arguments:
 *   cache  : may be NULL when the metadata has no cached segment; otherwise
 *            its segments must be exactly the metadata's cached layout
 *            (SCA_ERR_MISMATCH) and its heads the call's heads;
 *   md     : built and uploaded (sca_metadata_upload) before this call;
 *   q, k_cur, v_cur, o : bf16 token-major [n_queries][heads][128];
 *   lse    : fp32 [heads][n_queries] natural-log sum-exp, or NULL;
 *   workspace, workspace_bytes : optional device scratch (256-byte aligned).
 *            With enough of it (sca_attn_workspace_bytes) the work items
 *            left after the last full wave of SMs are split along the keys
 *            and merged by a second kernel, which removes the partial last
 *            wave; with NULL or too little, nothing is split. The result is
 *            the same up to fp32 summation order;
 *   dev_status : device int32 (or NULL); left unchanged on success, set to
 *            SCA_ERR_DEVICE_TIMEOUT if a bounded wait in the kernel ran out,
 *            or SCA_ERR_MISALIGNED if the kernel's shared-memory window did
 *            not start close enough to a 1024-byte boundary (the INT8 cache
 *            kernel has under 1 KB to spare; the result is then not written);
 *   stream : the caller's stream.
 * The call allocates nothing. A query that sees no key gets o = 0 and
 * lse = -inf. Calls sharing a workspace must be ordered (same stream). */
SCA_API int sca_action_causal_attn_fwd(const sca_kv_cache* cache, const sca_metadata* md,
                               int32_t heads, const void* q, const void* k_cur,
                               const void* v_cur, void* o, float* lse,
                               float softmax_scale, void* workspace, uint64_t workspace_bytes,
                               int32_t* dev_status, void* stream);

/* Workspace the attention would use on the current device for `heads` heads
 * (0 when the plan splits nothing). */
SCA_API int sca_attn_workspace_bytes(const sca_metadata* md, int32_t heads, uint64_t* bytes);

/* INT8 cache: extra workspace for a bf16 copy of the cached K and V
 * (2 · heads · n_cache · 256 bytes, each half 256-byte aligned). When the
 * workspace given to the attention holds sca_attn_workspace_bytes (rounded up
 * to 256) plus this, the call first dequantises the cache into it, once,
 * with an HBM-bound copy kernel, and runs the bf16 kernel on the copy;
 * otherwise the INT8 kernel dequantises tile by tile in shared memory, again
 * for every query-tile pair that reads the tile. Both paths feed the same
 * bf16 values to the products and give the same result bit for bit; the
 * persistent cache stays INT8 either way (a model's per-layer caches can
 * share one copy buffer). */
SCA_API int sca_attn_int8_scratch_bytes(const sca_metadata* md, int32_t heads, uint64_t* bytes);

/* The plan the next attention call with enough workspace would run: the
 * first n_full work items (query-tile pair x head) whole, the remaining
 * n_split items cut into `chunks` key ranges each. Any output may be NULL. */
SCA_API int sca_attn_plan(const sca_metadata* md, int32_t heads, int32_t* n_full,
                          int32_t* n_split, int32_t* chunks);

/* The plan (and its workspace bytes) for a device with `sms` SMs, without
 * touching any device: for planning ahead of a launch on another GPU, and
 * for host-only tests. sca_attn_plan gives the same result for the current
 * device's SM count. Honours sca_set_split_override. Any output may be NULL. */
SCA_API int sca_attn_plan_for_sms(const sca_metadata* md, int32_t heads, int32_t sms,
                                  int32_t* n_full, int32_t* n_split, int32_t* chunks,
                                  uint64_t* workspace_bytes);

/* Override of the key-split factor used by later attention calls made from
 * the calling host thread (other threads keep their own setting, so a test
 * or tuning loop on one thread cannot change another thread's calls):
 * 0 = automatic (default), 1 = never split, k >= 2 = split every work item
 * after the full waves into k chunks (a test and tuning knob). */
SCA_API int sca_set_split_override(int32_t chunks);

/* Limit, in nanoseconds, of every pipeline wait inside the kernels (for a
 * tile load, a product or a handshake between warps) of later attention calls
 * made from the calling host thread: [0, 10 s], default 2 s. A wait that runs
 * out stores SCA_ERR_DEVICE_TIMEOUT in the call's device status word and makes
 * every CTA of the kernel stop issuing work; the output is then undefined.
 * Before a CTA frees its tensor memory and exits, it still waits for the
 * loads and products it has already issued, with a fixed limit of its own
 * (2 s) that this setting does not change, so the device stays usable. A test
 * and debugging knob: 0 makes a call give up at its first wait that is not
 * complete at once, which exercises that abort path on the real kernels. */
SCA_API int sca_set_pipeline_timeout_ns(int64_t ns);

/* Attention forward for callers that cannot allocate device memory (no
 * counterpart in the Hy-Nomas pages; a deployment convenience). Some callers
 * must never call the allocator - a latency-bound inference loop (cudaMalloc
 * can synchronise the device or fail under memory pressure), or a host
 * runtime whose own allocator owns all device memory - and so cannot provide
 * the workspace sca_action_causal_attn_fwd takes for its key-split partials.
 * This variant computes exactly what sca_action_causal_attn_fwd computes with
 * a workspace, but takes the partials from a fixed array of
 * SCA_STATIC_WORKSPACE_BYTES that is part of the library; it allocates
 * nothing. Arguments and results are those of sca_action_causal_attn_fwd,
 * without the workspace.
 *   - Limit: the array holds 32 MiB, enough for the automatic split plans
 *     of the 480p single-turn and long-session layouts (16 heads; with or
 *     without a sliding window or a quarter of the video blocks) on a
 *     148-SM B200. If the automatic plan needs more (sca_attn_workspace_bytes;
 *     other layouts, other SM counts), the call runs every work item whole,
 *     which needs no scratch. If a split forced with sca_set_split_override
 *     needs more, it returns SCA_ERR_CAPACITY and launches nothing.
 *   - INT8 cache: when the split partials plus a bf16 copy of the cached K
 *     and V (sca_attn_int8_scratch_bytes) fit in the array, the call also
 *     dequantises the cache once into the array and runs the bf16 kernel on
 *     the copy, exactly as sca_action_causal_attn_fwd does with a workspace
 *     that large; otherwise it dequantises tile by tile. Same result.
 *   - Set-up: the first call on each device (with that device current) looks
 *     up the array's device address, once per context (again after a
 *     cudaDeviceReset); make that first call before any stream capture.
 *   - Sharing: every call, on every stream, uses the same array, which keeps
 *     the last call's contents. Nothing in it needs to start at zero (a call
 *     reads only partials and copies it wrote itself), but calls that
 *     overlap on the GPU race: order them (one stream, or events).
 *   - Memory: every GPU that loads the library holds the array until the
 *     process exits. */
#define SCA_STATIC_WORKSPACE_BYTES (32ull << 20)
SCA_API int sca_action_causal_attn_fwd_static_ws(const sca_kv_cache* cache,
                                                 const sca_metadata* md, int32_t heads,
                                                 const void* q, const void* k_cur,
                                                 const void* v_cur, void* o, float* lse,
                                                 float softmax_scale, int32_t* dev_status,
                                                 void* stream);

/* ---------------------------------------------------------------------------
 * Attention backward, for layouts without cached segments (the packed,
 * FLOPs-balanced training batches of the picx.dev summary, "Methodology ›
 * Training Infrastructure"; the pages print no backward pass, so its
 * gradients are those of the forward above). Per head, over the visible
 * pairs, with P the row softmax (recomputed from the forward's LSE):
 *   dV = Pᵀ dO,  dP = dO Vᵀ,  D_i = Σ_d dO_id O_id,  dS = P ∘ (dP − D),
 *   dQ = scale · dS K,  dK = scale · dSᵀ Q.
 * Arguments:
 *   md     : built and uploaded; no cached segments (SCA_ERR_UNSUPPORTED);
 *            the same layout, window and dropped blocks as the forward;
 *   q, k, v, o, d_o : bf16 token-major [n][heads][128], n = the metadata's
 *            queries (= keys): the forward's inputs, its output and dO;
 *   lse    : fp32 [heads][n], the forward's (natural log);
 *   dq, dk, dv : bf16 [n][heads][128], written (not accumulated);
 *   workspace, workspace_bytes : device scratch of at least
 *            sca_attn_bwd_workspace_bytes (256-byte aligned; required:
 *            SCA_ERR_CAPACITY otherwise); it receives −D and −LSE·log2(e);
 *   dev_status, stream : as for the forward.
 * Three kernels on the stream: D and LSE, dQ (query tiles over their key
 * tiles), dK and dV (key tiles over the query tiles that see them); no
 * atomics, so the result does not depend on scheduling. The call allocates
 * nothing. A key no query sees gets dK = dV = 0. The dK/dV kernel uses all
 * 227 KB of shared memory a CTA may have and needs its dynamic shared memory
 * to start on a 1024-byte boundary (as on B200); if it does not, the kernel
 * does nothing and writes SCA_ERR_MISALIGNED to dev_status. */
SCA_API int sca_action_causal_attn_bwd(const sca_metadata* md, int32_t heads, const void* q,
                                       const void* k, const void* v, const void* o,
                                       const float* lse, const void* d_o, void* dq, void* dk,
                                       void* dv, float softmax_scale, void* workspace,
                                       uint64_t workspace_bytes, int32_t* dev_status,
                                       void* stream);

/* Host view of the backward's key-major schedule (layouts without a cache;
 * empty otherwise): kt_ptr[n_kv_tiles + 1] and kt_list[nnz], for each key tile
 * the query tiles that see part of it in ascending order, each entry
 * query tile | class << 24 (the transpose of the CSR schedule above);
 * kt_order[n_kv_tiles], the key tiles most expensive first. Valid until the
 * next build or destroy; all three are NULL for a layout with a cache. Any
 * output may be NULL. */
SCA_API int sca_metadata_get_bwd_schedule(const sca_metadata* md, const int32_t** kt_ptr,
                                          const uint32_t** kt_list, const int32_t** kt_order);

/* Workspace the backward needs: 2 · heads · round_up(n, 128) floats. */
SCA_API int sca_attn_bwd_workspace_bytes(const sca_metadata* md, int32_t heads, uint64_t* bytes);

/* ---------------------------------------------------------------------------
 * Camera cross-attention of one segment: the attention core of Eq. 3 of
 * [picx.dev summary, Methodology › Model Architecture, Camera-Trajectory
 * Conditioning], V~ = V + CrossAttn(V, C), with the visual tokens as queries
 * and the segment's camera tokens (one per latent frame, aligned in time with
 * the frames [onedev.kr review, "어떻게 쓰나"]) as keys and values, on inputs
 * already projected per head (the projections are model weights):
 *
 *   out_i = x_i + sum_f softmax_f(softmax_scale · <q_i, k_f>) v_f
 *
 * over the camera tokens f that query i sees. The pages leave that set open
 * beyond "time-aligned"; `mode` picks a reading:
 *   SCA_CAM_ALL         every camera token of the segment;
 *   SCA_CAM_OWN_FRAME   only the token of the query's own latent frame;
 *   SCA_CAM_UP_TO_FRAME the tokens of latent frames 0 .. the query's own.
 * A query whose frame lies outside [0, n_cam) sees no token in the two
 * frame modes and keeps out_i = x_i.
 * Arguments:
 *   q, x, out : bf16 token-major [n_q][heads][128] (16-byte aligned); out
 *            may be x (the residual updated in place), no other overlap;
 *   q_frame : int32 [n_q], each query's latent frame in the segment; may be
 *            NULL for SCA_CAM_ALL;
 *   k_cam, v_cam : bf16 [n_cam][heads][128] (16-byte aligned);
 *   n_q >= 0, 1 <= n_cam <= SCA_MAX_CAMERA_TOKENS, heads >= 1;
 *   softmax_scale : finite (1/sqrt(128) for the model's heads);
 *   dev_status : device int32 (or NULL); left unchanged on success, set to
 *            SCA_ERR_DEVICE_TIMEOUT if a staged tile does not land within the
 *            pipeline-wait limit (sca_set_pipeline_timeout_ns), the output
 *            then incomplete.
 * S and O are accumulated in fp32, P is rounded to bf16 for its product, the
 * output is rounded once to bf16. Enqueued on `stream` as a programmatic
 * dependent launch: the kernel may start its set-up while earlier work on the
 * stream finishes, but reads and writes memory only after that work is
 * complete, so the ordering is that of a plain launch. Allocates nothing.
 * SCA_ERR_INVALID_ARG / SCA_ERR_MISALIGNED on bad arguments, and
 * SCA_ERR_UNSUPPORTED past 65,535 heads or 2^31 elements of q (nothing is
 * launched then). */
enum { SCA_CAM_ALL = 0, SCA_CAM_OWN_FRAME = 1, SCA_CAM_UP_TO_FRAME = 2 };
#define SCA_MAX_CAMERA_TOKENS 64
SCA_API int sca_camera_cross_attn(const void* q, const int32_t* q_frame, const void* k_cam,
                                  const void* v_cam, const void* x, void* out, int32_t n_q,
                                  int32_t n_cam, int32_t heads, int32_t mode,
                                  float softmax_scale, int32_t* dev_status, void* stream);

/* Message of the calling thread's last failure ("" if none). */
SCA_API const char* sca_last_error(void);

/* Read a device status word (the dev_status of the attention calls): waits
 * for the work queued on `stream` so far, copies the word to the host and
 * returns it: SCA_OK when no kernel reported a failure, else the negative
 * code a kernel stored (SCA_ERR_DEVICE_TIMEOUT, SCA_ERR_MISALIGNED), with a
 * message from sca_last_error. SCA_ERR_CUDA if the copy itself fails,
 * SCA_ERR_INVALID_ARG for a null pointer. The word is left as it is; the
 * caller clears it (a 4-byte memset) before reusing it. */
SCA_API int sca_read_device_status(const int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * Self-test of the device-side bounded wait: one block waits on an mbarrier
 * that nothing completes, gives up after `timeout_ns` nanoseconds, writes
 * SCA_ERR_DEVICE_TIMEOUT to *dev_status and returns. Exists so the timeout
 * path can be exercised without any real hang.
 * ------------------------------------------------------------------------- */
SCA_API int sca_debug_bounded_wait(int32_t* dev_status, int64_t timeout_ns, void* stream);


#ifdef __cplusplus
}
#endif

#endif /* SCA_H_ */
