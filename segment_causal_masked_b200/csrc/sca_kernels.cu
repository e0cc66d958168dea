// Device kernels of libsca for NVIDIA B200 (sm_100a):
//
//  * kv_append_kernel   - appends a segment's K/V to the head-major bf16 cache
//                         with 16-byte coalesced loads and stores and writes its
//                         key descriptors, tails marked dead (gpts24.com, "One
//                         World, Generated Segment by Segment"; picx.dev
//                         summary, "Action-Aware Causal Attention (Figure 6b)").
//  * attn_fwd_kernel    - flash-style forward of action-aware causal attention:
//                         TMA-staged Q/K/V tiles, tcgen05 MMAs accumulating in
//                         tensor memory (S = Q K^T and O += P V, P read from
//                         tensor memory), online softmax in fp32 with the mask
//                         evaluated from descriptor words on PARTIAL tiles only.
//  * bounded_wait_kernel - exercises the timeout path of the bounded mbarrier
//                         wait every pipeline wait here goes through.
//
// Attention CTA organisation (one CTA per (query-tile pair, head)):
//   warps 0-3  softmax of query tile 0 (one thread per row = TMEM lane)
//   warps 4-7  softmax of query tile 1
//   warp  8    TMA producer (Q once, then K_j, V_j into a 4-stage ring)
//   warp  9    TMEM allocator and MMA issuer (one elected thread)
//   warps 10-11 idle (they complete the control warpgroup's register split)
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0 [256,384),
// O1 [384,512); P_t (bf16 pairs) overwrites the first 64 columns of S_t.
// The MMA warp ping-pongs the two tiles: while softmax works on tile 0's
// scores the tensor cores run tile 1's P V and next S, and vice versa.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "sca_internal.h"
#include "sca_ptx.cuh"

namespace sca {

// ---------------------------------------------------------------------------
// kv_cache_append
// ---------------------------------------------------------------------------

// Descriptor word of every appended token (tails marked dead).
__device__ __forceinline__ void append_descriptors(const AppendArgs& a) {
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; t < a.n; t += stride) {
    uint32_t d;
    if (t < a.n_video) {
      d = a.seg_index | SCA_DESC_ALIVE;
    } else if (t < int64_t(a.n_video) + a.head_len) {
      d = a.seg_index | SCA_DESC_ALIVE | SCA_DESC_HEAD;
    } else {
      const int32_t r = int32_t(t - a.n_video - a.head_len);
      int act = 0;
      while (act + 1 < a.n_act && r >= a.tail_start[act + 1]) ++act;
      d = a.seg_index | SCA_DESC_TAIL | (uint32_t(act) << SCA_DESC_ACTION_SHIFT);  // dead later
    }
    a.desc[a.length + t] = d;
  }
}

__global__ void __launch_bounds__(256) kv_append_kernel(const AppendArgs a) {
  const uint4* __restrict__ k = static_cast<const uint4*>(a.k);
  const uint4* __restrict__ v = static_cast<const uint4*>(a.v);
  uint4* __restrict__ kc = static_cast<uint4*>(a.k_cache);
  uint4* __restrict__ vc = static_cast<uint4*>(a.v_cache);
  const int64_t per_tok = int64_t(a.heads) * 16;  // 16-byte chunks per token
  const int64_t total = int64_t(a.n) * per_tok;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int64_t tok = i / per_tok;
    const int32_t rem = int32_t(i - tok * per_tok);
    const int32_t h = rem >> 4, c = rem & 15;
    const int64_t dst = ((int64_t(h) * a.capacity) + a.length + tok) * 16 + c;
    const uint4 kk = __ldg(k + i);
    const uint4 vv = __ldg(v + i);
    kc[dst] = kk;
    vc[dst] = vv;
  }
  append_descriptors(a);
}

// Quantise one 128-value row spread over a warp (4 values per lane, given as
// two bf16 pairs): scale = max|x| / 127 and code = rint(x / scale) in fp32,
// both divisions correctly rounded and the rounding to nearest even, codes
// clamped to [-127, 127]; a zero row gets scale 0 and codes 0. Returns the
// lane's four codes as offset-binary bytes (code + 128), low byte first.
__device__ __forceinline__ uint32_t quantize_lane(uint2 raw, float& scale) {
  float x[4];
  x[0] = __uint_as_float(raw.x << 16);
  x[1] = __uint_as_float(raw.x & 0xFFFF0000u);
  x[2] = __uint_as_float(raw.y << 16);
  x[3] = __uint_as_float(raw.y & 0xFFFF0000u);
  float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
  scale = __fdiv_rn(amax, 127.f);
  uint32_t packed = 0x80808080u;  // code 0 in every byte
  if (scale > 0.f) {
    packed = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int qi = min(max(__float2int_rn(__fdiv_rn(x[i], scale)), -127), 127);
      packed |= uint32_t(qi + 128) << (8 * i);
    }
  }
  return packed;
}

// INT8 cache append: one warp per (token, head) row, K and V; 4-byte code
// stores (a row of codes is one coalesced 128-byte line).
__global__ void __launch_bounds__(256) kv_append_int8_kernel(const AppendArgs a) {
  const uint2* __restrict__ k = static_cast<const uint2*>(a.k);
  const uint2* __restrict__ v = static_cast<const uint2*>(a.v);
  uint32_t* __restrict__ kc = static_cast<uint32_t*>(a.k_cache);
  uint32_t* __restrict__ vc = static_cast<uint32_t*>(a.v_cache);
  const int lane = threadIdx.x & 31;
  const int64_t rows = int64_t(a.n) * a.heads;
  const int64_t wstride = int64_t(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += wstride) {
    const int64_t tok = row / a.heads;
    const int32_t h = int32_t(row - tok * a.heads);
    const int64_t dst = int64_t(h) * a.capacity + a.length + tok;  // row of the cache
    float sk, sv;
    const uint32_t qk = quantize_lane(__ldg(k + row * 32 + lane), sk);
    const uint32_t qv = quantize_lane(__ldg(v + row * 32 + lane), sv);
    kc[dst * 32 + lane] = qk;
    vc[dst * 32 + lane] = qv;
    if (lane == 0) {
      a.k_scale[dst] = sk;
      a.v_scale[dst] = sv;
    }
  }
  append_descriptors(a);
}

// INT8 cache -> bf16 copy [heads][n][128] (the scratch path of the
// attention): each thread turns 16 codes of one row into bf16 with the
// arithmetic of the attention kernel's own dequantisation (exact c from the
// pattern 2^23 + (c + 128), c * scale rounded to fp32, then to bf16), so both
// paths feed the products the same values bit for bit.
__global__ void __launch_bounds__(256) kv_dequant_kernel(const DequantArgs a) {
  const uint4* __restrict__ codes[2] = {static_cast<const uint4*>(a.k_codes),
                                        static_cast<const uint4*>(a.v_codes)};
  const float* __restrict__ scales[2] = {a.k_scale, a.v_scale};
  uint4* __restrict__ outs[2] = {static_cast<uint4*>(a.k_out), static_cast<uint4*>(a.v_out)};
  const int64_t per_tensor = int64_t(a.heads) * a.n * 8;  // 16-code chunks
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  const uint64_t off2 = f2(-8388736.f, -8388736.f);       // -(2^23 + 128)
  const uint64_t zero2 = f2(0.f, 0.f);
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < 2 * per_tensor; i += stride) {
    const int t = i >= per_tensor;
    const int64_t c = i - t * per_tensor;                  // chunk within the tensor
    const int64_t row = c >> 3;                            // head * n + token
    const int64_t h = row / a.n, tok = row - h * a.n;
    const int64_t src_row = h * a.capacity + tok;
    const float s = scales[t][src_row];
    const uint64_t s2 = f2(s, s);
    const uint4 w = __ldg(codes[t] + src_row * 8 + (c & 7));
    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
    uint32_t out[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const float f0 = __uint_as_float(__byte_perm(words[k], 0x4B000000u, 0x7540u + 2u * b));
        const float f1 = __uint_as_float(__byte_perm(words[k], 0x4B000000u, 0x7541u + 2u * b));
        float v0, v1;
        unf2(fma2(add2(f2(f0, f1), off2), s2, zero2), v0, v1);
        out[2 * k + b] = pack_bf16(v0, v1);
      }
    }
    outs[t][c * 2] = make_uint4(out[0], out[1], out[2], out[3]);
    outs[t][c * 2 + 1] = make_uint4(out[4], out[5], out[6], out[7]);
  }
}

cudaError_t launch_dequant(const DequantArgs& a, cudaStream_t stream) {
  if (a.n <= 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t work = 2 * int64_t(a.heads) * a.n * 8;
  int64_t blocks = (work + 255) / 256;
  blocks = blocks < int64_t(sms) * 8 ? blocks : int64_t(sms) * 8;
  kv_dequant_kernel<<<unsigned(blocks), 256, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream) {
  if (a.n <= 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t chunks = int64_t(a.n) * a.heads * 16;
  int64_t blocks = (chunks + 255) / 256;
  blocks = blocks < int64_t(sms) * 8 ? blocks : int64_t(sms) * 8;
  if (a.int8) {
    kv_append_int8_kernel<<<unsigned(blocks), 256, 0, stream>>>(a);
  } else {
    kv_append_kernel<<<unsigned(blocks), 256, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

// p = exp2(x * scale - m) for one row's 128 scores, summed into `acc` and
// written as bf16 pairs over the first 64 TMEM columns of the row's S (P
// chunk c lands in S chunk c/2, whose scores are already in registers).
__device__ __forceinline__ void exp_pack_store(const float (&x)[128], uint64_t scale2,
                                               uint64_t negm2, uint32_t tS, uint64_t (&acc)[2]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float x0, x1;
      unf2(fma2(f2(x[32 * c + 2 * i], x[32 * c + 2 * i + 1]), scale2, negm2), x0, x1);
      const float p0 = ex2(x0), p1 = ex2(x1);
      acc[i & 1] = add2(acc[i & 1], f2(p0, p1));
      pk[i] = pack_bf16(p0, p1);
    }
    tmem_st16(tS + uint32_t(c) * 16, pk);
  }
}

// INT8 cache: dequantise row r of a staged code tile (128 rows of 128
// offset-binary codes, 128-byte swizzle, as the tensor copy lays it out) into row r of a
// bf16 operand tile in the layout the tensor copy of a bf16 tile gives (two
// 64-column halves 16 KB apart, 128-byte swizzle). A code c becomes the exact
// float c through the bit pattern 2^23 + (c + 128), then c * scale is rounded
// once to fp32 and once to bf16. Both tiles start on 1024-byte boundaries,
// so the swizzle of row r XORs the 16-byte chunk index with r & 7.
__device__ __forceinline__ void dequant_row(const uint8_t* codes, float scale, uint8_t* tile, int r) {
  const uint32_t sw = uint32_t(r & 7);
  const uint64_t s2 = f2(scale, scale);
  const uint64_t off2 = f2(-8388736.f, -8388736.f);  // -(2^23 + 128)
  const uint64_t zero2 = f2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < 8; ++c) {  // codes of columns 16c .. 16c + 15
    const uint4 w = *reinterpret_cast<const uint4*>(codes + r * 128 + ((uint32_t(c) ^ sw) << 4));
    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
    uint32_t out[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t u = words[k];  // c + 128 in every byte (offset binary)
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const float f0 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540u + 2u * b));
        const float f1 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7541u + 2u * b));
        float v0, v1;
        unf2(fma2(add2(f2(f0, f1), off2), s2, zero2), v0, v1);
        out[2 * k + b] = pack_bf16(v0, v1);
      }
    }
    uint8_t* row = tile + (c >> 2) * (128 * 128) + r * 128;  // half c / 4
    const uint32_t ch = uint32_t(2 * (c & 3));
    *reinterpret_cast<uint4*>(row + ((ch ^ sw) << 4)) = make_uint4(out[0], out[1], out[2], out[3]);
    *reinterpret_cast<uint4*>(row + (((ch + 1u) ^ sw) << 4)) = make_uint4(out[4], out[5], out[6], out[7]);
  }
}

// ---------------------------------------------------------------------------
// attention forward
// ---------------------------------------------------------------------------

constexpr int kStages = 4;       // bf16 cache: K/V ring depth (the most any instantiation uses)
constexpr int kStagesInt8 = 3;   // INT8 cache: ring depth (room for the code slots)
constexpr int kCodeSlots = 4;    // INT8 cache: staged code tiles
__host__ __device__ constexpr int ring_stages(bool int8) { return int8 ? kStagesInt8 : kStages; }
static_assert(kStagesInt8 <= kStages, "the barrier map holds kStages ring slots");
constexpr int kThreads = 384;     // 3 warpgroups (bf16 cache)
constexpr int kThreadsInt8 = 512; // + a dequantising warpgroup (INT8 cache)
__host__ __device__ constexpr int threads_for(bool int8) { return int8 ? kThreadsInt8 : kThreads; }
// Registers are split per warpgroup with setmaxnreg: the launch reserves
// 384 x 168 = 64,512 (168 is the most a thread can get when three warps share
// an SM sub-partition's 16K registers); the two softmax warpgroups grow to 224
// (a row's 128 scores stay in registers) and the producer/MMA warpgroup
// shrinks to 56: 2 x 128 x 224 + 128 x 56 = 64,512.
constexpr int kRegsSoftmax = 224;
constexpr int kRegsControl = 56;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsControl == kThreads * 168,
              "the register split must add up to the launch's registers");
// INT8: 512 threads launch with 128 registers each; the softmax warpgroups
// grow to 216 and the control and dequantising warpgroups shrink to 40
// (2 x 128 x 216 + 2 x 128 x 40 = 512 x 128; the split ptxas fits without
// spilling).
constexpr int kRegsSoftmaxInt8 = 216;
constexpr int kRegsControlInt8 = 40;
constexpr int kRegsDequantInt8 = 40;
static_assert(2 * 128 * kRegsSoftmaxInt8 + 128 * (kRegsControlInt8 + kRegsDequantInt8) ==
                  kThreadsInt8 * 128,
              "the INT8 register split must add up to the launch's registers");
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kHalf = 128 * 64 * 2;  // one 128-row x 64-column bf16 box: 16 KB
constexpr uint32_t kTile = 2 * kHalf;     // 128 x 128 bf16: 32 KB
constexpr float kRescaleThreshold = 8.0f; // log2 units: p stays <= 2^8 between rescales

// shared-memory map (offsets from a 1024-aligned base)
constexpr uint32_t kOffQ = 0;                            // Q0, Q1
constexpr uint32_t kOffKV = 2 * kTile;                   // ring of K/V tiles
// INT8 cache only: kCodeSlots staged code tiles and their 128 row scales
constexpr uint32_t kCodeTile = 128 * 128;                // 16 KB
constexpr uint32_t kScaleBytes = 128 * 4;
__host__ __device__ constexpr uint32_t off_codes(bool int8) { return kOffKV + ring_stages(int8) * kTile; }
__host__ __device__ constexpr uint32_t off_scales(bool int8) { return off_codes(int8) + kCodeSlots * kCodeTile; }
__host__ __device__ constexpr uint32_t off_bar(bool int8) {
  return int8 ? off_scales(int8) + kCodeSlots * kScaleBytes : off_codes(int8);
}
constexpr uint32_t kBarQ = 0, kBarFull = 1, kBarEmpty = kBarFull + kStages,
                   kBarS = kBarEmpty + kStages, kBarP = kBarS + 2, kBarO = kBarP + 2,
                   kBarDrain = kBarO + 2, kBarCodeFull = kBarDrain + 1,
                   kBarCodeEmpty = kBarCodeFull + kCodeSlots, kNumBars = kBarCodeEmpty + kCodeSlots;
// The tiles need a 1024-byte aligned base. The dynamic shared window is
// padded so that the base can be moved up to the next boundary: by a full
// 1024 bytes when that fits the 227 KB a CTA may use (bf16), else by what is
// left (INT8, whose 4 code slots leave about 800 bytes). CUDA places the
// window on a 1024-byte boundary, so no padding is used in practice; a base
// the padding cannot fix makes the kernel report SCA_ERR_MISALIGNED.
constexpr uint32_t kSmemLimit = 232448;
__host__ __device__ constexpr uint32_t smem_used(bool int8) {
  return off_bar(int8) + kNumBars * 8 + 16 + 16;  // bars, control, TMEM slot
}
__host__ __device__ constexpr uint32_t align_slack(bool int8) {
  return kSmemLimit - smem_used(int8) < 1024 ? kSmemLimit - smem_used(int8) : 1024;
}
__host__ __device__ constexpr uint32_t smem_bytes(bool int8) { return smem_used(int8) + align_slack(int8); }
static_assert(smem_used(true) + 512 <= kSmemLimit, "the INT8 layout must fit the 227 KB a CTA may use");

size_t attention_smem_bytes(bool int8_cache) { return smem_bytes(int8_cache); }

// kInt8: the cache holds int8 codes with per-row scales (tm_kcache and
// tm_vcache cover the codes, tm_kscale and tm_vscale the scales); a fourth
// warpgroup dequantises the cache tiles into the operand ring ahead of the
// MMAs. Otherwise the cache is bf16 and the scale maps are unused.
template <bool kInt8>
__global__ void __launch_bounds__(threads_for(kInt8), 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_kcur,
                    const __grid_constant__ CUtensorMap tm_vcur,
                    const __grid_constant__ CUtensorMap tm_kcache,
                    const __grid_constant__ CUtensorMap tm_vcache,
                    const __grid_constant__ CUtensorMap tm_kscale,
                    const __grid_constant__ CUtensorMap tm_vscale, const AttnArgs p) {
  constexpr int kRing = ring_stages(kInt8);
  constexpr uint32_t kOffCodes = off_codes(kInt8), kOffScales = off_scales(kInt8);
  constexpr uint32_t kOffBar = off_bar(kInt8);
  constexpr uint32_t kOffCtl = kOffBar + kNumBars * 8;
  constexpr uint32_t kOffTmemSlot = kOffCtl + 16;
  extern __shared__ uint8_t smem_raw[];
  if ((1024u - (smem_u32(smem_raw) & 1023u)) % 1024u > align_slack(kInt8)) {
    // the padding does not reach the next 1024-byte boundary: report
    // instead of running misaligned (never taken with the full 1024)
    if (threadIdx.x == 0 && p.status) atomicExch(p.status, SCA_ERR_MISALIGNED);
    return;
  }
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kOffBar;
  auto bar = [&](uint32_t i) { return bar0 + 8 * i; };
  volatile Ctl* ctl = reinterpret_cast<volatile Ctl*>(smem + kOffCtl);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffTmemSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // which work item (query-tile pair x head), and which of its key tiles
  int item = int(blockIdx.x), chunk = 0, slot = -1;
  if (item >= p.n_full) {  // a key chunk of a split item (chunk-major order)
    const int u = item - p.n_full;
    chunk = u / p.n_split;
    const int si = u - chunk * p.n_split;
    item = p.n_full + si;
    slot = si * p.chunks + chunk;
  }
  const int rank = item / p.heads;
  const int head = item - rank * p.heads;
  const int pair = p.item_order[rank];
  const int pair_len = p.pair_ptr[pair + 1] - p.pair_ptr[pair];
  const int j_begin = int((int64_t(pair_len) * chunk) / p.chunks);
  const int j_end = slot < 0 ? pair_len : int((int64_t(pair_len) * (chunk + 1)) / p.chunks);
  const int n_iter = j_end - j_begin;
  const uint32_t* list = p.pair_list + p.pair_ptr[pair] + j_begin;
  const int q_row0 = pair * 256;

  if (threadIdx.x == 0) {
    ctl->abort = 0;
    mbar_init(bar(kBarQ), 1);
    for (int s = 0; s < kRing; ++s) {
      // INT8: a dequantised tile is complete after its warpgroup's 128 arrivals
      mbar_init(bar(kBarFull + s), kInt8 ? 128 : 1);
      mbar_init(bar(kBarEmpty + s), 1);
    }
    for (int s = 0; s < kCodeSlots; ++s) {
      mbar_init(bar(kBarCodeFull + s), 1);
      mbar_init(bar(kBarCodeEmpty + s), 128);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(kBarS + t), 1);
      mbar_init(bar(kBarP + t), 128);
      mbar_init(bar(kBarO + t), 1);
    }
    mbar_init(bar(kBarDrain), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
  if (kInt8 && warp >= 12) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsDequantInt8));
    // ------------------------------------------------------------ dequantiser
    // INT8 cache: thread r converts row r of every cache tile of the list (K
    // and V alternate; the cache tiles are a prefix of the ascending list)
    // from its staged code slot into the operand ring, as soon as the codes
    // have landed and the ring slot is free.
    const int r = int(threadIdx.x) - 384;
    for (int it = 0; it < 2 * n_iter; ++it) {
      if (int(list[it >> 1] & kPairTileMask) >= p.n_cache_tiles) break;
      const int slot8 = it % kCodeSlots, s = it % kRing;
      const bool ready = wait_bar(bar(kBarCodeFull + slot8), uint32_t(it / kCodeSlots) & 1u, ctl,
                                  p.status, p.timeout_ns) &&
                         wait_bar(bar(kBarEmpty + s), (uint32_t(it / kRing) & 1u) ^ 1u, ctl,
                                  p.status, p.timeout_ns);
      if (!__all_sync(0xFFFFFFFFu, ready)) break;
      const float sc = reinterpret_cast<const float*>(smem + kOffScales + slot8 * kScaleBytes)[r];
      dequant_row(smem + kOffCodes + slot8 * kCodeTile, sc, smem + kOffKV + s * kTile, r);
      fence_proxy_async_smem();
      mbar_arrive(bar(kBarFull + s));
      mbar_arrive(bar(kBarCodeEmpty + slot8));
    }
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kInt8 ? kRegsControlInt8 : kRegsControl));
  if (warp >= 10) {
    // warps 10-11 only complete the control warpgroup
  } else if (warp == kLoadWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_iter > 0) {
      const uint32_t sQ = sbase + kOffQ;
      mbar_expect_tx(bar(kBarQ), 2 * kTile);
      tma_load_3d(sQ, &tm_q, bar(kBarQ), 0, head, q_row0);
      tma_load_3d(sQ + kHalf, &tm_q, bar(kBarQ), 64, head, q_row0);
      tma_load_3d(sQ + kTile, &tm_q, bar(kBarQ), 0, head, q_row0 + 128);
      tma_load_3d(sQ + kTile + kHalf, &tm_q, bar(kBarQ), 64, head, q_row0 + 128);
      int it = 0;
      bool ok = true;
      // INT8: the cache tiles (a prefix of the ascending list) go to the code
      // slots, where a softmax warpgroup dequantises them into the ring
      auto staged = [&](int i) { return kInt8 && int(list[i >> 1] & kPairTileMask) < p.n_cache_tiles; };
      for (int j = 0; j < n_iter && ok; ++j) {
        const int tile = int(list[j] & kPairTileMask);
        for (int kv = 0; kv < 2; ++kv, ++it) {
          if (staged(it)) {
            const int cs = it % kCodeSlots;
            const uint32_t cb = bar(kBarCodeFull + cs);
            if (!wait_bar(bar(kBarCodeEmpty + cs), (uint32_t(it / kCodeSlots) & 1u) ^ 1u, ctl,
                          p.status, p.timeout_ns)) {
              ok = false;
              break;
            }
            mbar_expect_tx(cb, kCodeTile + kScaleBytes);
            tma_load_3d(sbase + kOffCodes + uint32_t(cs) * kCodeTile, kv ? &tm_vcache : &tm_kcache,
                        cb, 0, tile * 128, head);
            tma_load_2d(sbase + kOffScales + uint32_t(cs) * kScaleBytes,
                        kv ? &tm_vscale : &tm_kscale, cb, tile * 128, head);
            continue;
          }
          if (kInt8 && it > 0 && staged(it - 1)) {
            // first direct load after the staged prefix: wait until every
            // staged tile is dequantised. Ring slots of the prefix were
            // claimed by the dequantiser, so their release barriers may lag
            // this thread's count by more than one phase, which a parity
            // wait cannot tell apart; once the prefix is done they cannot.
            for (int i2 = it - kCodeSlots < 0 ? 0 : it - kCodeSlots; i2 < it && ok; ++i2)
              ok = wait_bar(bar(kBarCodeEmpty + i2 % kCodeSlots), uint32_t(i2 / kCodeSlots) & 1u, ctl,
                            p.status, p.timeout_ns);
            if (!ok) break;
          }
          const int s = it % kRing;
          const uint32_t ph = uint32_t(it / kRing) & 1u;
          if (!wait_bar(bar(kBarEmpty + s), ph ^ 1u, ctl, p.status, p.timeout_ns)) {
            ok = false;
            break;
          }
          const uint32_t dst = sbase + kOffKV + uint32_t(s) * kTile;
          mbar_expect_tx(bar(kBarFull + s), kTile);
          if (kInt8) mbar_arrive_n(bar(kBarFull + s), 127);
          if (!kInt8 && tile < p.n_cache_tiles) {
            const CUtensorMap* m = kv ? &tm_vcache : &tm_kcache;
            tma_load_3d(dst, m, bar(kBarFull + s), 0, tile * 128, head);
            tma_load_3d(dst + kHalf, m, bar(kBarFull + s), 64, tile * 128, head);
          } else {
            const CUtensorMap* m = kv ? &tm_vcur : &tm_kcur;
            const int row = (tile - p.n_cache_tiles) * 128;
            tma_load_3d(dst, m, bar(kBarFull + s), 0, head, row);
            tma_load_3d(dst + kHalf, m, bar(kBarFull + s), 64, head, row);
          }
        }
      }
      // Drain, also after a normal end (where it finds every load landed):
      // every armed load lands before the CTA can exit, even when a consumer
      // gave up and will never wait for it. The latest load of each ring
      // slot is among the last kRing issued (the staged loads among them
      // filled no ring slot); that of each code slot among the last
      // kCodeSlots staged loads, which form a prefix.
      for (int back = 1; back <= kRing && it - back >= 0; ++back) {
        const int i2 = it - back;
        if (!staged(i2)) wait_drain(bar(kBarFull + i2 % kRing), uint32_t(i2 / kRing) & 1u);
      }
      int n_staged = 0;
      while (n_staged < it && staged(n_staged)) ++n_staged;
      for (int i2 = n_staged - kCodeSlots < 0 ? 0 : n_staged - kCodeSlots; i2 < n_staged; ++i2)
        wait_drain(bar(kBarCodeFull + i2 % kCodeSlots), uint32_t(i2 / kCodeSlots) & 1u);
      wait_drain(bar(kBarQ), 0);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_iter > 0) {
      const uint32_t sQ0 = sbase + kOffQ, sQ1 = sQ0 + kTile;
      const uint32_t tS0 = tmem, tS1 = tmem + 128, tO0 = tmem + 256, tO1 = tmem + 384;
      auto issue_qk = [&](uint32_t tS, uint32_t sQ, uint32_t sK) {
        mma_qk8(tS, desc_kmajor(sQ), desc_kmajor(sK), kIdescQK);
      };
      auto issue_pv = [&](uint32_t tO, uint32_t tP, uint32_t sV, bool acc) {
        mma_pv8(tO, tP, desc_mnmajor(sV), kIdescPV, acc ? 1u : 0u);
      };
      auto stage_of = [&](int it) { return sbase + kOffKV + uint32_t(it % kRing) * kTile; };
      auto wait_full = [&](int it) {
        return wait_bar(bar(kBarFull + it % kRing), uint32_t(it / kRing) & 1u, ctl, p.status,
                        p.timeout_ns);
      };
      // a tile of the pair that sees nothing of key tile j gets neither its
      // S nor its P V; its barriers still complete (a commit with nothing
      // new arrives once the earlier MMAs are done)
      // (schedule entries of key tiles j and j + 1 stay in registers; the
      // entry of j + 2 is fetched one step ahead, off the issue path)
      auto live = [&](uint32_t e, int t) { return ((e >> (24 + 2 * t)) & 3u) != SCA_TILE_EMPTY; };
      uint32_t e_cur = list[0];
      uint32_t e_nxt = n_iter > 1 ? list[1] : 0u;
      bool acc0 = false, acc1 = false;  // has O_t received a P V yet
      bool ok = wait_bar(bar(kBarQ), 0, ctl, p.status, p.timeout_ns) && wait_full(0);
      if (ok) {
        tc_fence_after();
        if (live(e_cur, 0)) issue_qk(tS0, sQ0, stage_of(0));
        mma_commit(bar(kBarS + 0));
        if (live(e_cur, 1)) issue_qk(tS1, sQ1, stage_of(0));
        mma_commit(bar(kBarS + 1));
        mma_commit(bar(kBarEmpty + 0));
      }
      for (int j = 0; j < n_iter && ok; ++j) {
        const int itV = 2 * j + 1, itK = 2 * j + 2;
        const uint32_t ph = uint32_t(j) & 1u;
        const bool more = j + 1 < n_iter;
        const uint32_t e_after = j + 2 < n_iter ? list[j + 2] : 0u;
        // K of the next tile first, so that P V and the next S go out back to back
        ok = wait_full(itV) && (!more || wait_full(itK)) &&
             wait_bar(bar(kBarP + 0), ph, ctl, p.status, p.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        if (live(e_cur, 0)) {
          issue_pv(tO0, tS0, stage_of(itV), acc0);
          acc0 = true;
        }
        if (more) {
          if (live(e_nxt, 0)) issue_qk(tS0, sQ0, stage_of(itK));
          mma_commit(bar(kBarS + 0));
        }
        if (!(ok = wait_bar(bar(kBarP + 1), ph, ctl, p.status, p.timeout_ns))) break;
        tc_fence_after();
        if (live(e_cur, 1)) {
          issue_pv(tO1, tS1, stage_of(itV), acc1);
          acc1 = true;
        }
        mma_commit(bar(kBarEmpty + itV % kRing));
        if (more) {
          if (live(e_nxt, 1)) issue_qk(tS1, sQ1, stage_of(itK));
          mma_commit(bar(kBarS + 1));
          mma_commit(bar(kBarEmpty + itK % kRing));
        }
        e_cur = e_nxt;
        e_nxt = e_after;
      }
      mma_commit(bar(kBarO + 0));
      mma_commit(bar(kBarO + 1));
      // every MMA has finished before this thread leaves (also on abort)
      mma_commit(bar(kBarDrain));
      wait_drain(bar(kBarDrain), 0);
    }
    __syncwarp();
  }
  }
  } else {
    // ------------------------------------------------------------ softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kInt8 ? kRegsSoftmaxInt8 : kRegsSoftmax));
    const int t = warp >> 2;           // query tile of the pair
    const int wq = warp & 3;           // TMEM lane quadrant
    const int r = wq * 32 + lane;      // row in the tile
    const int q_row = q_row0 + t * 128 + r;
    const uint2 qd = p.qdesc[q_row];
    const uint32_t lane_base = tmem + (uint32_t(wq * 32) << 16);
    const uint32_t tS = lane_base + uint32_t(t) * 128;
    const uint32_t tO = lane_base + 256 + uint32_t(t) * 128;
    float m_run = -INFINITY, l_run = 0.f;
    bool o_init = false;  // O_t holds a P V result (else its TMEM is undefined)
    bool ok = true;
    const uint64_t scale2 = f2(p.scale_log2, p.scale_log2);
    uint32_t e_next = n_iter > 0 ? list[0] : 0u;
    for (int j = 0; j < n_iter; ++j) {
      const uint32_t e = e_next;
      if (j + 1 < n_iter) e_next = list[j + 1];   // prefetch the next schedule entry
      const int tile = int(e & kPairTileMask);
      const uint32_t cls = (e >> (24 + 2 * t)) & 3u;
      // PARTIAL: this row's visibility of the tile's 128 columns, one
      // predicate per run of equal key descriptors (computed before waiting
      // for S so it overlaps the MMA); columns past the source are in no run.
      uint32_t vis[4] = {0u, 0u, 0u, 0u};
      if (cls == SCA_TILE_PARTIAL) {
        const int r0 = p.run_ptr[tile], r1 = p.run_ptr[tile + 1];
        for (int i = r0; i < r1; ++i) {
          const uint2 run = p.runs[i];
          if (!visible(qd.x, qd.y, run.y, uint32_t(p.history))) continue;
          const int a = int(run.x & 255u), b = a + int((run.x >> 8) & 255u);
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int lo = max(a, 32 * w) - 32 * w, hi = min(b, 32 * w + 32) - 32 * w;
            if (lo < hi) vis[w] |= uint32_t(((1ull << (hi - lo)) - 1ull) << lo);
          }
        }
      }
      ok = wait_bar(bar(kBarS + t), uint32_t(j) & 1u, ctl, p.status, p.timeout_ns);
      if (!__all_sync(0xFFFFFFFFu, ok)) {  // keep the warp's collective TMEM ops uniform
        ok = false;
        break;
      }
      tc_fence_after();
      if (cls == SCA_TILE_EMPTY) {
        // this tile sees nothing of key tile j: the MMA warp issued neither
        // its S nor its P V, nothing to do but keep the handshake
      } else {
        // One pass: all 128 scores of the row come out of TMEM with four
        // loads in flight and a single wait.
        float x[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + uint32_t(c) * 32, x + 32 * c);
        tmem_wait_ld();
        if (cls == SCA_TILE_PARTIAL) {
#pragma unroll
          for (int i = 0; i < 128; ++i) x[i] = ((vis[i >> 5] >> (i & 31)) & 1u) ? x[i] : -INFINITY;
        }
        // row max in four chains: x[0..3], then x[4..123] two at a time,
        // then x[124..127]
        float m4[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
        for (int i = 4; i < 124; i += 8) {
#pragma unroll
          for (int k = 0; k < 4; ++k) m4[k] = max3(m4[k], x[i + k], x[i + 4 + k]);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) m4[k] = fmaxf(m4[k], x[124 + k]);
        const float mx = max3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
        // The running max only moves when it grows by more than the threshold
        // (exact: l and O share the stale max until the final division).
        // rounded on its own (no FMA with the subtraction below), so that
        // every instantiation of this kernel takes the same alpha
        const float m_cand = __fmul_rn(mx, p.scale_log2);
        const bool grow = m_cand > m_run + kRescaleThreshold;
        const bool rescale = grow && m_run != -INFINITY && o_init;
        const float alpha = rescale ? ex2(m_run - m_cand) : 1.f;
        if (grow) m_run = m_cand;
        const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
        const uint64_t negm2 = f2(neg_m, neg_m);
        uint64_t acc[2] = {0ull, 0ull};  // packed partial sums
        // p = exp2(s * scale_log2 - m), row sum, bf16 P
        exp_pack_store(x, scale2, negm2, tS, acc);
        float a0, a1;
        unf2(add2(acc[0], acc[1]), a0, a1);
        // one explicit rounding (l alpha + sum), so every instantiation of
        // this kernel gives the same l, whatever the compiler would contract
        l_run = fmaf(l_run, alpha, a0 + a1);
        // Rescale O. tcgen05.ld/st are warp-collective: the whole warp
        // rewrites O if any row needs it (alpha = 1 for the others). O of
        // earlier tiles was complete when S of this tile completed (in-order
        // MMA pipeline); P*V of this tile waits for the arrive below.
        if (__any_sync(0xFFFFFFFFu, rescale)) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float o[32];
            tmem_ld32(tO + uint32_t(c) * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tO + uint32_t(c) * 32, o);
          }
        }
        o_init = true;  // the P V of this tile will initialise / update O
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kBarP + t));
    }
    // ---------------------------------------------------------- epilogue
    if (ok && n_iter > 0) ok = wait_bar(bar(kBarO + t), 0, ctl, p.status, p.timeout_ns);
    if (__all_sync(0xFFFFFFFFu, ok)) {
      tc_fence_after();
      const bool store = q_row < p.n_q;
      if (slot >= 0) {
        // partial of a split item: unnormalised O, running max and sum (log2)
        const int prow = t * 128 + r;
        float4* po = reinterpret_cast<float4*>(p.part_o + (int64_t(slot) * 256 + prow) * 128);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float o[32];
          if (n_iter > 0) {
            tmem_ld32(tO + uint32_t(c) * 32, o);
            tmem_wait_ld();
          }
          if (!(n_iter > 0 && o_init && l_run > 0.f)) {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0.f;
          }
          if (store) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              po[c * 8 + i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
          }
        }
        if (store) p.part_ml[int64_t(slot) * 256 + prow] = make_float2(m_run, l_run);
      } else {
        const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
        uint4* orow = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) +
                                               (int64_t(q_row) * p.heads + head) * 128);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float o[32];
          if (n_iter > 0) {
            tmem_ld32(tO + uint32_t(c) * 32, o);
            tmem_wait_ld();
          }
          if (!(n_iter > 0 && o_init && l_run > 0.f)) {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0.f;
          }
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = pack_bf16(o[2 * i] * inv_l, o[2 * i + 1] * inv_l);
          if (store) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              orow[c * 4 + i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          }
        }
        if (store && p.lse)
          p.lse[int64_t(head) * p.n_q + q_row] =
              l_run > 0.f ? (m_run + __log2f(l_run)) * 0.6931471805599453f : -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

template <bool kInt8>
static cudaError_t launch_attention_t(const AttnMaps& maps, const AttnArgs& args,
                                      cudaStream_t stream) {
  // devices whose kernel attributes are set (a set bit; set at most once
  // per device, safely from several host threads)
  static std::atomic<uint32_t> configured_mask{0u};
  constexpr uint32_t kSmem = smem_bytes(kInt8);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 31 || !(configured_mask.load() & (1u << dev))) {
    e = cudaFuncSetAttribute(attn_fwd_kernel<kInt8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(kSmem));
    if (e != cudaSuccess) return e;
    if (dev < 31) configured_mask.fetch_or(1u << dev);
  }
  const unsigned grid = unsigned(args.n_full) + unsigned(args.n_split) * unsigned(args.chunks);
  attn_fwd_kernel<kInt8><<<grid, threads_for(kInt8), kSmem, stream>>>(
      maps.q, maps.k_cur, maps.v_cur, maps.k_cache, maps.v_cache, maps.k_scale, maps.v_scale, args);
  return cudaGetLastError();
}

cudaError_t launch_attention(const AttnMaps& maps, const AttnArgs& args, bool int8_cache,
                             cudaStream_t stream) {
  return int8_cache ? launch_attention_t<true>(maps, args, stream)
                    : launch_attention_t<false>(maps, args, stream);
}

// ---------------------------------------------------------------------------
// merge of the key chunks of split items
// ---------------------------------------------------------------------------

// One warp per query row of a split item (32 CTAs of 8 warps per item): with
// chunk maxima m_k and sums l_k (log2 domain) and unnormalised O_k,
//   M = max m_k,  w_k = 2^(m_k - M),  O = sum w_k O_k / sum w_k l_k,
//   LSE = (M + log2 sum w_k l_k) ln 2.
// A chunk that saw no key has l_k = 0 and O_k = 0 (the attention kernel
// stores zeros then), so it gets weight 0 and its loads need no branch.
__global__ void __launch_bounds__(256) merge_kernel(const AttnArgs p) {
  const int si = blockIdx.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int prow = (blockIdx.x & 31) * 8 + warp;
  const int item = p.n_full + si;
  const int rank = item / p.heads;
  const int head = item - rank * p.heads;
  const int pair = p.item_order[rank];
  const int q_row = pair * 256 + prow;
  if (q_row >= p.n_q) return;
  const int64_t slot0 = int64_t(si) * p.chunks;
  float M = -INFINITY;
#pragma unroll 8
  for (int k = 0; k < p.chunks; ++k) {
    const float2 ml = p.part_ml[(slot0 + k) * 256 + prow];
    M = ml.y > 0.f ? fmaxf(M, ml.x) : M;
  }
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float L = 0.f;
#pragma unroll 8
  for (int k = 0; k < p.chunks; ++k) {
    const float2 ml = p.part_ml[(slot0 + k) * 256 + prow];
    const float4 v = reinterpret_cast<const float4*>(p.part_o + ((slot0 + k) * 256 + prow) * 128)[lane];
    const float w = ml.y > 0.f ? ex2(ml.x - M) : 0.f;
    L += w * ml.y;
    acc.x += w * v.x;
    acc.y += w * v.y;
    acc.z += w * v.z;
    acc.w += w * v.w;
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  uint2 out;
  out.x = pack_bf16(acc.x * inv, acc.y * inv);
  out.y = pack_bf16(acc.z * inv, acc.w * inv);
  reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.o) +
                           (int64_t(q_row) * p.heads + head) * 128)[lane] = out;
  if (lane == 0 && p.lse)
    p.lse[int64_t(head) * p.n_q + q_row] =
        L > 0.f ? (M + __log2f(L)) * 0.6931471805599453f : -INFINITY;
}

cudaError_t launch_merge(const AttnArgs& args, cudaStream_t stream) {
  if (args.n_split <= 0) return cudaSuccess;
  merge_kernel<<<unsigned(args.n_split) * 32u, 256, 0, stream>>>(args);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// bounded-wait self-test
// ---------------------------------------------------------------------------

__global__ void bounded_wait_kernel(int32_t* status, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t never;
  __shared__ Ctl ctl;
  if (threadIdx.x == 0) {
    ctl.abort = 0;
    mbar_init(smem_u32(&never), 1);  // nobody ever arrives
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) wait_bounded(smem_u32(&never), 0, &ctl, status, timeout_ns);
}

cudaError_t launch_bounded_wait(int32_t* status, unsigned long long timeout_ns,
                                cudaStream_t stream) {
  bounded_wait_kernel<<<1, 32, 0, stream>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace sca
