// Attention backward of libsca for NVIDIA B200 (sm_100a): dQ, dK, dV of the
// action-aware causal attention for layouts without cached segments (the
// packed training batches of [picx.dev summary, Methodology › Training
// Infrastructure]). Per head, with P the row softmax of the visible scores
// (recomputed from the forward's LSE), D_i = Σ_d dO_id O_id and
// dS = P ∘ (dO Vᵀ − D):  dV = Pᵀ dO,  dQ = scale · dS K,  dK = scale · dSᵀ Q.
//
// Three kernels, one stream:
//   bwd_prep_kernel   D and LSE·log2(e) per (head, query) into the workspace;
//   bwd_dq_kernel     one CTA per (query tile, head), over the query tile's
//                     key tiles: S = Q Kᵀ and dP = dO Vᵀ into TMEM, dS in
//                     registers, dQ += dS K accumulated in TMEM;
//   bwd_dkdv_kernel   one CTA per (key tile, head), over the query tiles that
//                     see it: Sᵀ = K Qᵀ and dPᵀ = V dOᵀ into TMEM, Pᵀ and dSᵀ
//                     (bf16) back into TMEM, dV += Pᵀ dO and dK += dSᵀ Q.
// S and dP are computed twice (once per kernel) so that neither dQ nor dK/dV
// needs atomics. The schedules are the forward's tile classes: the dQ kernel
// reads the pair work list, the dK/dV kernel its transpose (per key tile, the
// query tiles with their classes); PARTIAL tiles are masked with the same
// predicate on descriptor words, per run of equal descriptors.
//
// Warp roles (384 threads, as in the forward): warps 0-3 and 4-7 do the
// elementwise work of columns 0-63 and 64-127 of every row (one thread per
// TMEM lane, so no row needs a reduction: D and the LSE are precomputed);
// warp 8 issues the TMA loads; warp 9 allocates TMEM and issues the MMAs;
// warp 10 issues the dP products (dQ kernel) or the dO loads (dK/dV kernel).

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "sca_internal.h"
#include "sca_ptx.cuh"

namespace sca {

namespace {

constexpr int kBThreads = 384;
constexpr int kBRegsWork = 224;
constexpr int kBRegsControl = 56;
static_assert(2 * 128 * kBRegsWork + 128 * kBRegsControl == kBThreads * 168,
              "the register split must add up to the launch's registers");
constexpr uint32_t kBHalf = 128 * 64 * 2;  // 128 rows x 64 bf16 columns
constexpr uint32_t kBTile = 2 * kBHalf;    // 128 x 128 bf16
constexpr float kLog2e = 1.4426950408889634f;

// D (+)= A B with A from TMEM as two 32-column halves (keys or queries 0-63 at
// a_lo, 64-127 at a_hi; 8 columns per K-step of 16) and B MN-major in shared
// memory (2048 B per K-step). `acc` = 0 overwrites D on the first step.
__device__ __forceinline__ void mma_ts8_split(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi,
                                              uint64_t b_desc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred pf, pt;\n\t.reg .b32 ta, bl;\n\t.reg .b64 bd;\n\t"
      "setp.ne.b32 pf, %6, 0;\n\tsetp.eq.b32 pt, 0, 0;\n\t"
      "mov.b64 bd, {%3, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], bd, %5, pf;\n\t"
      "add.u32 ta, %1, 8;\n\tadd.u32 bl, %3, 128;\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %5, pt;\n\t"
      "add.u32 ta, %1, 16;\n\tadd.u32 bl, %3, 256;\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %5, pt;\n\t"
      "add.u32 ta, %1, 24;\n\tadd.u32 bl, %3, 384;\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %5, pt;\n\t"
      "add.u32 bl, %3, 512;\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], bd, %5, pt;\n\t"
      "add.u32 ta, %2, 8;\n\tadd.u32 bl, %3, 640;\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %5, pt;\n\t"
      "add.u32 ta, %2, 16;\n\tadd.u32 bl, %3, 768;\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %5, pt;\n\t"
      "add.u32 ta, %2, 24;\n\tadd.u32 bl, %3, 896;\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %5, pt;\n\t}"
      ::"r"(d_tmem), "r"(a_lo), "r"(a_hi), "r"(uint32_t(b_desc)), "r"(uint32_t(b_desc >> 32)),
      "r"(idesc), "r"(acc)
      : "memory");
}

// D (+)= A B with A from TMEM laid out by the dK/dV kernel: the 16-query
// K-step k sits at column a + {0, 8, 32, 40, 16, 24, 48, 56}[k] (warpgroup
// (k/2) % 2 wrote queries [64 b, 64 b + 64) of its 32-column blocks at
// 32 w + 16 b); B MN-major, 2048 B per K-step.
__device__ __forceinline__ void mma_ts8_blocks(uint32_t d_tmem, uint32_t a, uint64_t b_desc,
                                               uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred pf, pt;\n\t.reg .b32 ta, bl;\n\t.reg .b64 bd;\n\t"
      "setp.ne.b32 pf, %5, 0;\n\tsetp.eq.b32 pt, 0, 0;\n\t"
      "mov.b64 bd, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], bd, %4, pf;\n\t"
      "add.u32 ta, %1, 8;\n\tadd.u32 bl, %2, 128;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %4, pt;\n\t"
      "add.u32 ta, %1, 32;\n\tadd.u32 bl, %2, 256;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %4, pt;\n\t"
      "add.u32 ta, %1, 40;\n\tadd.u32 bl, %2, 384;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %4, pt;\n\t"
      "add.u32 ta, %1, 16;\n\tadd.u32 bl, %2, 512;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %4, pt;\n\t"
      "add.u32 ta, %1, 24;\n\tadd.u32 bl, %2, 640;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %4, pt;\n\t"
      "add.u32 ta, %1, 48;\n\tadd.u32 bl, %2, 768;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %4, pt;\n\t"
      "add.u32 ta, %1, 56;\n\tadd.u32 bl, %2, 896;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %4, pt;\n\t}"
      ::"r"(d_tmem), "r"(a), "r"(uint32_t(b_desc)), "r"(uint32_t(b_desc >> 32)), "r"(idesc),
      "r"(acc)
      : "memory");
}

// Columns [c0, c0 + 32) of a run [a, b) as a 32-bit mask.
__device__ __forceinline__ uint32_t run_bits32(int a, int b, int c0) {
  const int lo = max(a, c0) - c0, hi = min(b, c0 + 32) - c0;
  return lo < hi ? uint32_t(((1ull << (hi - lo)) - 1ull) << lo) : 0u;
}

// Columns [c0, c0 + 64) of a run [a, b) as two 32-bit masks.
__device__ __forceinline__ void set_run_bits(uint32_t (&vis)[2], int a, int b, int c0) {
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    const int lo = max(a, c0 + 32 * w) - (c0 + 32 * w);
    const int hi = min(b, c0 + 32 * w + 32) - (c0 + 32 * w);
    if (lo < hi) vis[w] |= uint32_t(((1ull << (hi - lo)) - 1ull) << lo);
  }
}

// ds = p (dp - d) with p = exp2(s * scale_log2 - l) where visible (0
// elsewhere), for 32 columns given as pairs; nl2 = (-l, -l), nd2 = (-d, -d)
// per column pair. Packed fp32 pairs; bf16 pairs of ds out.
template <bool kFull>
__device__ __forceinline__ void ds_pairs(const float (&s)[32], const float (&dp)[32],
                                         uint32_t vis, uint64_t c2, const uint64_t* nl2,
                                         const uint64_t* nd2, uint32_t (&dsw)[16],
                                         uint32_t* pw = nullptr) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float x0, x1;
    unf2(fma2(f2(s[2 * i], s[2 * i + 1]), c2, nl2[i]), x0, x1);
    float p0 = ex2(x0), p1 = ex2(x1);
    if (!kFull) {
      p0 = ((vis >> (2 * i)) & 1u) ? p0 : 0.f;
      p1 = ((vis >> (2 * i + 1)) & 1u) ? p1 : 0.f;
    }
    const uint64_t pp = f2(p0, p1);
    float d0, d1;
    unf2(mul2(pp, add2(f2(dp[2 * i], dp[2 * i + 1]), nd2[i])), d0, d1);
    dsw[i] = pack_bf16(d0, d1);
    if (pw) pw[i] = pack_bf16(p0, p1);
  }
}

// The two halves of ds_pairs, for a caller that stores P before it has dP:
// p = 2^(s · scale_log2 − L), masked like ds_pairs, in place, with its bf16
// pairs in pw ...
template <bool kFull>
__device__ __forceinline__ void p_pairs(float (&s)[32], uint32_t vis, uint64_t c2,
                                        const uint64_t* nl2, uint32_t (&pw)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float x0, x1;
    unf2(fma2(f2(s[2 * i], s[2 * i + 1]), c2, nl2[i]), x0, x1);
    float p0 = ex2(x0), p1 = ex2(x1);
    if (!kFull) {
      p0 = ((vis >> (2 * i)) & 1u) ? p0 : 0.f;
      p1 = ((vis >> (2 * i + 1)) & 1u) ? p1 : 0.f;
    }
    s[2 * i] = p0;
    s[2 * i + 1] = p1;
    pw[i] = pack_bf16(p0, p1);
  }
}

// ... and then dS = P ∘ (dP − D) as bf16 pairs (the same operations, in the
// same order, as ds_pairs)
__device__ __forceinline__ void ds_from_p(const float (&p)[32], const float (&dp)[32],
                                          const uint64_t* nd2, uint32_t (&dsw)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float d0, d1;
    unf2(mul2(f2(p[2 * i], p[2 * i + 1]), add2(f2(dp[2 * i], dp[2 * i + 1]), nd2[i])), d0, d1);
    dsw[i] = pack_bf16(d0, d1);
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// D = rowsum(dO ∘ O) and LSE · log2(e), per (head, query)
// ---------------------------------------------------------------------------

// One warp per (query, head) row, 4 values per lane; the workspace receives
// -D and -L (L = LSE · log2 e). Rows past n (up to the tile-padded n_pad) get
// 0; the kernels never use them unmasked. A row with LSE = -inf (it sees
// nothing) gets L = +inf, so that its probabilities come out 0.
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdArgs a) {
  const uint2* __restrict__ o = static_cast<const uint2*>(a.o);
  const uint2* __restrict__ g = static_cast<const uint2*>(a.d_o);
  const int lane = threadIdx.x & 31;
  const int64_t rows = int64_t(a.n_pad) * a.heads;
  const int64_t wstride = int64_t(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += wstride) {
    const int64_t tok = row / a.heads;
    const int h = int(row - tok * a.heads);
    float d = 0.f, l = 0.f;
    if (tok < a.n) {
      const uint2 x = __ldg(o + row * 32 + lane);
      const uint2 y = __ldg(g + row * 32 + lane);
      d = __uint_as_float(x.x << 16) * __uint_as_float(y.x << 16) +
          __uint_as_float(x.x & 0xFFFF0000u) * __uint_as_float(y.x & 0xFFFF0000u) +
          __uint_as_float(x.y << 16) * __uint_as_float(y.y << 16) +
          __uint_as_float(x.y & 0xFFFF0000u) * __uint_as_float(y.y & 0xFFFF0000u);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xFFFFFFFFu, d, off);
      const float lse = a.lse[int64_t(h) * a.n + tok];
      l = lse == -INFINITY ? INFINITY : lse * kLog2e;
    }
    if (lane == 0) {  // stored negated: the kernels add them with packed FMAs
      a.dl[int64_t(h) * a.n_pad + tok] = -d;
      a.dl[int64_t(a.heads + h) * a.n_pad + tok] = -l;
    }
  }
}

// ---------------------------------------------------------------------------
// dQ
// ---------------------------------------------------------------------------

// shared memory (1024-aligned base): Q, dO, a ring of 3 K tiles and one of 2
// V tiles (K_j is read by S_j and, a step later, by dQ += dS_j K_j).
constexpr uint32_t kQOffQ = 0, kQOffDO = kBTile, kQOffK = 2 * kBTile, kQOffV = 5 * kBTile;
constexpr int kQKSlots = 3, kQVSlots = 2;
constexpr uint32_t kQBarQD = 0, kQBarKF = 1, kQBarKE = kQBarKF + kQKSlots,
                   kQBarVF = kQBarKE + kQKSlots, kQBarVE = kQBarVF + kQVSlots,
                   kQBarS = kQBarVE + kQVSlots, kQBarDP = kQBarS + 2, kQBarDS = kQBarDP + 1,
                   kQBarRD = kQBarDS + 2, kQBarDone = kQBarRD + 1, kQBarDrain = kQBarDone + 1,
                   kQBarDrainP = kQBarDrain + 1, kQNumBars = kQBarDrainP + 1;
// dS barriers alternate by step parity: the elementwise warps can finish step
// j + 1 before the MMA thread has seen step j (the next dP starts on the
// read-done signal), and a single barrier could then run two phases ahead
// of the MMA thread's parity wait.
constexpr uint32_t kQOffBar = 7 * kBTile;
constexpr uint32_t kQOffCtl = kQOffBar + kQNumBars * 8;
constexpr uint32_t kQOffSlot = kQOffCtl + 16;
constexpr uint32_t kQSmem = kQOffSlot + 16 + 1024;
static_assert(kQSmem <= 232448, "the dQ kernel must fit the 227 KB a CTA may use");

__global__ void __launch_bounds__(kBThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_do, const BwdArgs p) {
  const int head = int(blockIdx.x) % p.heads;
  const int rest = int(blockIdx.x) / p.heads;
  const int t = rest & 1;                        // which tile of the pair
  const int pair = p.item_order[rest >> 1];
  const int qtile = 2 * pair + t;
  if (qtile >= p.n_q_tiles) return;              // the odd last pair has one tile
  const uint32_t* list = p.pair_list + p.pair_ptr[pair];
  const int len = p.pair_ptr[pair + 1] - p.pair_ptr[pair];
  auto cls_of = [&](int e) { return (list[e] >> (24 + 2 * t)) & 3u; };

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](uint32_t i) { return sbase + kQOffBar + 8 * i; };
  volatile Ctl* ctl = reinterpret_cast<volatile Ctl*>(smem + kQOffCtl);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kQOffSlot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    ctl->abort = 0;
    mbar_init(bar(kQBarQD), 1);
    for (int s = 0; s < kQKSlots; ++s) {
      mbar_init(bar(kQBarKF + s), 1);
      mbar_init(bar(kQBarKE + s), 1);
    }
    for (int s = 0; s < kQVSlots; ++s) {
      mbar_init(bar(kQBarVF + s), 1);
      mbar_init(bar(kQBarVE + s), 1);
    }
    mbar_init(bar(kQBarS), 1);
    mbar_init(bar(kQBarS + 1), 1);
    mbar_init(bar(kQBarDP), 1);
    mbar_init(bar(kQBarDS), 256);
    mbar_init(bar(kQBarDS + 1), 256);
    mbar_init(bar(kQBarRD), 256);
    mbar_init(bar(kQBarDone), 1);
    mbar_init(bar(kQBarDrain), 1);
    mbar_init(bar(kQBarDrainP), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS0 = tmem, tDP = tmem + 256, tDQ = tmem + 384;

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kBRegsControl));
    if (warp == 8 && lane == 0) {
      // ---------------------------------------------------------------- producer
      mbar_expect_tx(bar(kQBarQD), 2 * kBTile);
      const int q0 = qtile * 128;
      tma_load_3d(sbase + kQOffQ, &tm_q, bar(kQBarQD), 0, head, q0);
      tma_load_3d(sbase + kQOffQ + kBHalf, &tm_q, bar(kQBarQD), 64, head, q0);
      tma_load_3d(sbase + kQOffDO, &tm_do, bar(kQBarQD), 0, head, q0);
      tma_load_3d(sbase + kQOffDO + kBHalf, &tm_do, bar(kQBarQD), 64, head, q0);
      int j = 0;
      bool ok = true;
      for (int e = 0; e < len && ok; ++e) {
        if (cls_of(e) == SCA_TILE_EMPTY) continue;
        const int row = int(list[e] & kPairTileMask) * 128;
        const int ks = j % kQKSlots, vs = j % kQVSlots;
        ok = wait_bar(bar(kQBarKE + ks), (uint32_t(j / kQKSlots) & 1u) ^ 1u, ctl, p.status,
                      p.timeout_ns);
        if (!ok) break;
        mbar_expect_tx(bar(kQBarKF + ks), kBTile);
        tma_load_3d(sbase + kQOffK + ks * kBTile, &tm_k, bar(kQBarKF + ks), 0, head, row);
        tma_load_3d(sbase + kQOffK + ks * kBTile + kBHalf, &tm_k, bar(kQBarKF + ks), 64, head, row);
        ok = wait_bar(bar(kQBarVE + vs), (uint32_t(j / kQVSlots) & 1u) ^ 1u, ctl, p.status,
                      p.timeout_ns);
        if (!ok) {
          wait_drain(bar(kQBarKF + ks), uint32_t(j / kQKSlots) & 1u);  // this K load is armed
          break;
        }
        mbar_expect_tx(bar(kQBarVF + vs), kBTile);
        tma_load_3d(sbase + kQOffV + vs * kBTile, &tm_v, bar(kQBarVF + vs), 0, head, row);
        tma_load_3d(sbase + kQOffV + vs * kBTile + kBHalf, &tm_v, bar(kQBarVF + vs), 64, head, row);
        ++j;
      }
      // Drain, also after a normal end (where it finds every load landed):
      // every armed load lands before the CTA can exit, even when a consumer
      // gave up (the latest load of each slot is among the last kQKSlots /
      // kQVSlots)
      for (int i = j - kQKSlots < 0 ? 0 : j - kQKSlots; i < j; ++i)
        wait_drain(bar(kQBarKF + i % kQKSlots), uint32_t(i / kQKSlots) & 1u);
      for (int i = j - kQVSlots < 0 ? 0 : j - kQVSlots; i < j; ++i)
        wait_drain(bar(kQBarVF + i % kQVSlots), uint32_t(i / kQVSlots) & 1u);
      wait_drain(bar(kQBarQD), 0);
    } else if (warp == 9 || warp == 10) {
      // ---------------------------------------------------------------- MMA
      // Two issuing threads, so that neither product stream waits behind the
      // other's barrier: warp 9 issues S = Q Kᵀ and dQ += dS K, warp 10 the
      // dP = dO Vᵀ products (on disjoint TMEM columns and operands; each
      // thread's commits track its own products).
      int n = 0;  // live key tiles of this query tile, counted by the warp
      for (int e0 = 0; e0 < len; e0 += 32) {
        const bool live = e0 + lane < len && cls_of(e0 + lane) != SCA_TILE_EMPTY;
        n += __popc(__ballot_sync(0xFFFFFFFFu, live));
      }
      if (lane == 0) {
        const uint64_t dQ = desc_kmajor(sbase + kQOffQ), dDO = desc_kmajor(sbase + kQOffDO);
        auto kslot = [&](int j) { return sbase + kQOffK + uint32_t(j % kQKSlots) * kBTile; };
        auto vslot = [&](int j) { return sbase + kQOffV + uint32_t(j % kQVSlots) * kBTile; };
        auto wait_k = [&](int j) {
          return wait_bar(bar(kQBarKF + j % kQKSlots), uint32_t(j / kQKSlots) & 1u, ctl, p.status,
                          p.timeout_ns);
        };
        auto wait_v = [&](int j) {
          return wait_bar(bar(kQBarVF + j % kQVSlots), uint32_t(j / kQVSlots) & 1u, ctl, p.status,
                          p.timeout_ns);
        };
        auto issue_dp = [&](int j) {  // dP_j = dO V_jᵀ; the last read of V_j
          mma_qk8(tDP, dDO, desc_kmajor(vslot(j)), kIdescQK);
          mma_commit(bar(kQBarDP));
          mma_commit(bar(kQBarVE + j % kQVSlots));
        };
        // Q and dO are always loaded: wait for them even with no key tile
        bool ok = wait_bar(bar(kQBarQD), 0, ctl, p.status, p.timeout_ns);
        if (warp == 9) {
          if (ok && n > 0 && (ok = wait_k(0))) {
            tc_fence_after();
            mma_qk8(tS0, dQ, desc_kmajor(kslot(0)), kIdescQK);
            mma_commit(bar(kQBarS));
          }
          if (ok && n > 1 && (ok = wait_k(1))) {
            tc_fence_after();
            mma_qk8(tS0 + 128, dQ, desc_kmajor(kslot(1)), kIdescQK);
            mma_commit(bar(kQBarS + 1));
          }
          for (int j = 0; ok && j < n; ++j) {
            const uint32_t tSj = tS0 + uint32_t(j & 1) * 128;
            if (!(ok = wait_bar(bar(kQBarDS + (j & 1)), uint32_t(j >> 1) & 1u, ctl, p.status,
                                p.timeout_ns)))
              break;
            tc_fence_after();
            mma_ts8_split(tDQ, tSj, tSj + 64, desc_mnmajor(kslot(j)), kIdescPV, j > 0 ? 1u : 0u);
            mma_commit(bar(kQBarKE + j % kQKSlots));
            if (j + 2 < n) {  // S of the key tile after next into the slot dS_j leaves
              if (!(ok = wait_k(j + 2))) break;
              tc_fence_after();
              mma_qk8(tSj, dQ, desc_kmajor(kslot(j + 2)), kIdescQK);
              mma_commit(bar(kQBarS + (j & 1)));
            }
          }
          mma_commit(bar(kQBarDone));
          mma_commit(bar(kQBarDrain));
          wait_drain(bar(kQBarDrain), 0);
        } else {
          if (ok && n > 0 && (ok = wait_v(0))) {
            tc_fence_after();
            issue_dp(0);
          }
          // dP of the next key tile as soon as dP_j has been read out: it
          // overlaps the elementwise work on this one
          for (int j = 0; ok && j + 1 < n; ++j) {
            if (!(ok = wait_bar(bar(kQBarRD), uint32_t(j) & 1u, ctl, p.status, p.timeout_ns) &&
                       wait_v(j + 1)))
              break;
            tc_fence_after();
            issue_dp(j + 1);
          }
          mma_commit(bar(kQBarDrainP));
          wait_drain(bar(kQBarDrainP), 0);
        }
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------------ elementwise
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kBRegsWork));
    const int half = warp >> 2;                   // columns [64 half, 64 half + 64)
    const int r = (warp & 3) * 32 + lane;         // row = TMEM lane
    const int q_row = qtile * 128 + r;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint2 qd = p.qdesc[q_row];
    const float nl = p.dl[int64_t(p.heads + head) * p.n_pad + q_row];  // -L
    const float nd = p.dl[int64_t(head) * p.n_pad + q_row];            // -D
    uint64_t nl2[16], nd2[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      nl2[i] = f2(nl, nl);
      nd2[i] = f2(nd, nd);
    }
    const uint64_t c2 = f2(p.scale_log2, p.scale_log2);
    const int c0 = 64 * half;
    bool ok = true;
    int j = 0;
    uint32_t e_next = len > 0 ? list[0] : 0u;
    for (int e = 0; e < len; ++e) {
      const uint32_t entry = e_next;
      if (e + 1 < len) e_next = list[e + 1];   // prefetch the next schedule entry
      const uint32_t cls = (entry >> (24 + 2 * t)) & 3u;
      if (cls == SCA_TILE_EMPTY) continue;
      const int tile = int(entry & kPairTileMask);
      uint32_t vis[2] = {0u, 0u};
      if (cls == SCA_TILE_PARTIAL) {
        for (int i = p.run_ptr[tile]; i < p.run_ptr[tile + 1]; ++i) {
          const uint2 run = p.runs[i];
          if (!visible(qd.x, qd.y, run.y, uint32_t(p.history))) continue;
          const int a = int(run.x & 255u);
          set_run_bits(vis, a, a + int((run.x >> 8) & 255u), c0);
        }
      }
      ok = wait_bar(bar(kQBarS + (j & 1)), uint32_t(j >> 1) & 1u, ctl, p.status, p.timeout_ns) &&
           wait_bar(bar(kQBarDP), uint32_t(j) & 1u, ctl, p.status, p.timeout_ns);
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tSj = tS0 + uint32_t(j & 1) * 128 + lane_base;
      float s[64], dp[64];
      tmem_ld32(tSj + c0, s);
      tmem_ld32(tSj + c0 + 32, s + 32);
      tmem_ld32(tDP + lane_base + c0, dp);
      tmem_ld32(tDP + lane_base + c0 + 32, dp + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(kQBarRD));  // dP_j is in registers: the next dP may overwrite it
      uint32_t dsw[32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float(&sh)[32] = *reinterpret_cast<const float(*)[32]>(s + 32 * h);
        const float(&dph)[32] = *reinterpret_cast<const float(*)[32]>(dp + 32 * h);
        uint32_t(&out)[16] = *reinterpret_cast<uint32_t(*)[16]>(dsw + 16 * h);
        if (cls == SCA_TILE_FULL) ds_pairs<true>(sh, dph, 0u, c2, nl2, nd2, out);
        else ds_pairs<false>(sh, dph, vis[h], c2, nl2, nd2, out);
      }
      tmem_st16(tSj + c0, dsw);  // dS over the first 32 columns of this half
      tmem_st16(tSj + c0 + 16, dsw + 16);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kQBarDS + (j & 1)));
      ++j;
    }
    // epilogue: dQ row (this half) = scale * accumulated dS K
    if (ok) ok = wait_bar(bar(kQBarDone), 0, ctl, p.status, p.timeout_ns);
    if (__all_sync(0xFFFFFFFFu, ok)) {
      tc_fence_after();
      float g[64];
      if (j > 0) {
        tmem_ld32(tDQ + lane_base + c0, g);
        tmem_ld32(tDQ + lane_base + c0 + 32, g + 32);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) g[i] = 0.f;
      }
      if (q_row < p.n) {
        uint4* out = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dq) +
                                              (int64_t(q_row) * p.heads + head) * 128 + c0);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          out[i] = make_uint4(pack_bf16(g[8 * i] * p.scale, g[8 * i + 1] * p.scale),
                              pack_bf16(g[8 * i + 2] * p.scale, g[8 * i + 3] * p.scale),
                              pack_bf16(g[8 * i + 4] * p.scale, g[8 * i + 5] * p.scale),
                              pack_bf16(g[8 * i + 6] * p.scale, g[8 * i + 7] * p.scale));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// ---------------------------------------------------------------------------
// dK and dV
// ---------------------------------------------------------------------------

// shared memory, from a 1024-aligned base: the barriers in the first 1 KB,
// then K and V of the CTA's key tile, a ring of 3 Q tiles and a ring of 2
// (dO tile, −D[128], −L[128]) stages (32 KB and 33 KB, so every tile stays
// 1024-aligned): 227 KB, all a CTA may have, so there is no room to align
// the base by hand and the kernel checks that it is aligned. Q_i is read by
// Sᵀ_i and again by dK += dSᵀ_i Q_i a query tile later, while Sᵀ of the
// next query tile is wanted early, so Q gets the deeper ring.
constexpr uint32_t kKBarKV = 0, kKBarQF = 1, kKQSlots = 3, kKBarQE = kKBarQF + kKQSlots,
                   kKOSlots = 2, kKBarOF = kKBarQE + kKQSlots, kKBarOE = kKBarOF + kKOSlots,
                   kKBarST = kKBarOE + kKOSlots, kKBarDPT = kKBarST + 1, kKBarRD = kKBarDPT + 1,
                   kKBarPR = kKBarRD + 1, kKBarDS = kKBarPR + 1, kKBarDone = kKBarDS + 1,
                   kKBarDrain = kKBarDone + 1, kKNumBars = kKBarDrain + 1;
constexpr uint32_t kKOffBar = 0;
constexpr uint32_t kKOffCtl = kKOffBar + kKNumBars * 8;
constexpr uint32_t kKOffSlot = kKOffCtl + 16;
constexpr uint32_t kKOffK = 1024, kKOffV = kKOffK + kBTile, kKOffQ = kKOffV + kBTile;
constexpr uint32_t kKOStage = kBTile + 1024;  // dO, −D[128], −L[128]
constexpr uint32_t kKOffO = kKOffQ + kKQSlots * kBTile;
constexpr uint32_t kKSmem = kKOffO + kKOSlots * kKOStage;
static_assert(kKOffSlot + 16 <= kKOffK, "the barriers fit the first 1 KB");
static_assert(kKSmem <= 232448, "the dK/dV kernel must fit the 227 KB a CTA may use");

// TMEM of the dK/dV kernel: two 128-column regions X and Y that swap roles
// every query tile, then dV and dK. Query tile i computes Sᵀ_i into
// region(i), overwrites it with Pᵀ_i (columns 0-63) and dSᵀ_i (64-127) for
// dV and dK, and takes dPᵀ_i in region(i + 1); so Sᵀ_{i+1} may start as soon
// as dPᵀ_i has been read out, while dV and dK of tile i still read region(i),
// and dPᵀ_{i+1} goes into region(i) once they have.
__global__ void __launch_bounds__(kBThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dl, const BwdArgs p) {
  const int head = int(blockIdx.x) % p.heads;
  const int ktile = p.kt_order[int(blockIdx.x) / p.heads];
  const uint32_t* list = p.kt_list + p.kt_ptr[ktile];
  const int n = p.kt_ptr[ktile + 1] - p.kt_ptr[ktile];

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {  // the layout needs a 1024-aligned base (uniform: all threads leave)
    if (threadIdx.x == 0 && p.status) atomicExch(p.status, SCA_ERR_MISALIGNED);
    return;
  }
  auto bar = [&](uint32_t i) { return sbase + kKOffBar + 8 * i; };
  auto qslot = [&](int i) { return sbase + kKOffQ + uint32_t(i % kKQSlots) * kBTile; };
  auto oslot = [&](int i) { return sbase + kKOffO + uint32_t(i % kKOSlots) * kKOStage; };
  volatile Ctl* ctl = reinterpret_cast<volatile Ctl*>(smem + kKOffCtl);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kKOffSlot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    ctl->abort = 0;
    mbar_init(bar(kKBarKV), 1);
    for (int s = 0; s < kKQSlots; ++s) {
      mbar_init(bar(kKBarQF + s), 1);
      mbar_init(bar(kKBarQE + s), 1);
    }
    for (int s = 0; s < kKOSlots; ++s) {
      mbar_init(bar(kKBarOF + s), 1);
      mbar_init(bar(kKBarOE + s), 1);
    }
    mbar_init(bar(kKBarST), 1);
    mbar_init(bar(kKBarDPT), 1);
    mbar_init(bar(kKBarRD), 256);
    mbar_init(bar(kKBarPR), 256);
    mbar_init(bar(kKBarDS), 256);
    mbar_init(bar(kKBarDone), 1);
    mbar_init(bar(kKBarDrain), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tDV = tmem + 256, tDK = tmem + 384;
  auto region = [&](int i) { return tmem + uint32_t(i & 1) * 128; };

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kBRegsControl));
    if (warp == 8 && lane == 0) {
      // ------------------------------------------------------ producer: K, V, Q
      const int k0 = ktile * 128;
      mbar_expect_tx(bar(kKBarKV), 2 * kBTile);
      tma_load_3d(sbase + kKOffK, &tm_k, bar(kKBarKV), 0, head, k0);
      tma_load_3d(sbase + kKOffK + kBHalf, &tm_k, bar(kKBarKV), 64, head, k0);
      tma_load_3d(sbase + kKOffV, &tm_v, bar(kKBarKV), 0, head, k0);
      tma_load_3d(sbase + kKOffV + kBHalf, &tm_v, bar(kKBarKV), 64, head, k0);
      int i = 0;
      for (; i < n; ++i) {
        const int s = i % kKQSlots;
        if (!wait_bar(bar(kKBarQE + s), (uint32_t(i / kKQSlots) & 1u) ^ 1u, ctl, p.status,
                      p.timeout_ns))
          break;
        const int q0 = int(list[i] & kPairTileMask) * 128;
        mbar_expect_tx(bar(kKBarQF + s), kBTile);
        tma_load_3d(qslot(i), &tm_q, bar(kKBarQF + s), 0, head, q0);
        tma_load_3d(qslot(i) + kBHalf, &tm_q, bar(kKBarQF + s), 64, head, q0);
      }
      // Drain, also after a normal end: every armed load lands before the
      // CTA can exit, even when a consumer gave up.
      for (int i2 = i - kKQSlots < 0 ? 0 : i - kKQSlots; i2 < i; ++i2)
        wait_drain(bar(kKBarQF + i2 % kKQSlots), uint32_t(i2 / kKQSlots) & 1u);
      wait_drain(bar(kKBarKV), 0);
    } else if (warp == 10 && lane == 0) {
      // ------------------------------------------------------ producer: dO
      int i = 0;
      for (; i < n; ++i) {
        const int s = i % kKOSlots;
        if (!wait_bar(bar(kKBarOE + s), (uint32_t(i / kKOSlots) & 1u) ^ 1u, ctl, p.status,
                      p.timeout_ns))
          break;
        const int q0 = int(list[i] & kPairTileMask) * 128;
        mbar_expect_tx(bar(kKBarOF + s), kKOStage);
        tma_load_3d(oslot(i), &tm_do, bar(kKBarOF + s), 0, head, q0);
        tma_load_3d(oslot(i) + kBHalf, &tm_do, bar(kKBarOF + s), 64, head, q0);
        tma_load_2d(oslot(i) + kBTile, &tm_dl, bar(kKBarOF + s), q0, head);
        tma_load_2d(oslot(i) + kBTile + 512, &tm_dl, bar(kKBarOF + s), q0, p.heads + head);
      }
      for (int i2 = i - kKOSlots < 0 ? 0 : i - kKOSlots; i2 < i; ++i2)
        wait_drain(bar(kKBarOF + i2 % kKOSlots), uint32_t(i2 / kKOSlots) & 1u);
    } else if (warp == 9 && lane == 0) {
      // ---------------------------------------------------------------- MMA
      const uint64_t dK = desc_kmajor(sbase + kKOffK), dV = desc_kmajor(sbase + kKOffV);
      auto wait_q = [&](int i) {
        return wait_bar(bar(kKBarQF + i % kKQSlots), uint32_t(i / kKQSlots) & 1u, ctl, p.status,
                        p.timeout_ns);
      };
      auto wait_o = [&](int i) {
        return wait_bar(bar(kKBarOF + i % kKOSlots), uint32_t(i / kKOSlots) & 1u, ctl, p.status,
                        p.timeout_ns);
      };
      auto issue_s = [&](int i) {  // Sᵀ_i = K Q_iᵀ into region(i)
        mma_qk8(region(i), dK, desc_kmajor(qslot(i)), kIdescQK);
        mma_commit(bar(kKBarST));
      };
      auto issue_dp = [&](int i) {  // dPᵀ_i = V dO_iᵀ into region(i + 1)
        mma_qk8(region(i + 1), dV, desc_kmajor(oslot(i)), kIdescQK);
        mma_commit(bar(kKBarDPT));
      };
      // K and V are always loaded: wait for them even with no query tile
      bool ok = wait_bar(bar(kKBarKV), 0, ctl, p.status, p.timeout_ns) &&
                (n == 0 || (wait_q(0) && wait_o(0)));
      if (ok && n > 0) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
      }
      for (int i = 0; ok && i < n; ++i) {
        const bool more = i + 1 < n;
        // Pᵀ_i stored (waited first: the elementwise warps cannot store Pᵀ_{i+1}
        // before Sᵀ_{i+1} below, so this barrier is never a phase ahead)
        if (!(ok = wait_bar(bar(kKBarPR), uint32_t(i) & 1u, ctl, p.status, p.timeout_ns))) break;
        // Sᵀ_{i+1} into the other region as soon as dPᵀ_i has been read out,
        // ahead of dV in the pipe: the next query tile's elementwise work
        // waits on it, while dV is needed only before the next dV
        if (more) {
          if (!(ok = wait_bar(bar(kKBarRD), uint32_t(i) & 1u, ctl, p.status, p.timeout_ns) &&
                     wait_q(i + 1)))
            break;
          tc_fence_after();
          issue_s(i + 1);
        }
        // dV += Pᵀ_i dO_i (B MN-major: rows are queries)
        tc_fence_after();
        mma_ts8_blocks(tDV, region(i), desc_mnmajor(oslot(i)), kIdescPV, i > 0 ? 1u : 0u);
        // dK += dSᵀ_i Q_i, then dPᵀ_{i+1} into region(i) right behind it (the
        // next dO stage is waited for first, so the two go out back to back;
        // the in-order pipe runs dPᵀ after dV and dK have read the region)
        if (!(ok = (!more || wait_o(i + 1)) &&
                   wait_bar(bar(kKBarDS), uint32_t(i) & 1u, ctl, p.status, p.timeout_ns)))
          break;
        tc_fence_after();
        mma_ts8_blocks(tDK, region(i) + 64, desc_mnmajor(qslot(i)), kIdescPV, i > 0 ? 1u : 0u);
        mma_commit(bar(kKBarQE + i % kKQSlots));  // the last read of Q_i
        // the dO stage too: dV has read dO_i and the elementwise warps their
        // −D and −L before arriving on dSᵀ
        mma_commit(bar(kKBarOE + i % kKOSlots));
        if (more) issue_dp(i + 1);
      }
      mma_commit(bar(kKBarDone));
      mma_commit(bar(kKBarDrain));
      wait_drain(bar(kKBarDrain), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ elementwise
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kBRegsWork));
    const int half = warp >> 2;                   // query blocks [32 half, +32), [64 + 32 half, +32)
    const int r = (warp & 3) * 32 + lane;         // key row = TMEM lane
    const int key = ktile * 128 + r;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t kd = p.kdesc[key];
    const int c0 = 64 * half;                     // output columns of this half (epilogue)
    const uint64_t c2 = f2(p.scale_log2, p.scale_log2);
    bool ok = true;
    int i = 0;
    uint32_t e_next = n > 0 ? list[0] : 0u;
    for (; i < n; ++i) {
      const uint32_t e = e_next;
      if (i + 1 < n) e_next = list[i + 1];     // prefetch the next schedule entry
      const int qt = int(e & kPairTileMask);
      const uint32_t cls = e >> 24;
      uint32_t vis[2] = {0u, 0u};  // query blocks b = 0, 1
      if (cls == SCA_TILE_PARTIAL && key < p.n) {  // a padding key sees nothing
        for (int k = p.qrun_ptr[qt]; k < p.qrun_ptr[qt + 1]; ++k) {
          const uint4 run = p.qruns[k];
          if (!visible(run.y, run.z, kd, uint32_t(p.history))) continue;
          const int a = int(run.x & 255u), b = a + int((run.x >> 8) & 255u);
          vis[0] |= run_bits32(a, b, 32 * half);
          vis[1] |= run_bits32(a, b, 64 + 32 * half);
        }
      }
      const uint32_t tR = region(i) + lane_base, tD = region(i + 1) + lane_base;
      // per query column −D and −L as pairs, from the dO stage; block b
      // covers queries [64 b + 32 half, +32) (16-byte broadcast loads: four
      // columns each)
      const uint8_t* ost = smem + kKOffO + uint32_t(i % kKOSlots) * kKOStage;
      const ulonglong2* ndq = reinterpret_cast<const ulonglong2*>(ost + kBTile);
      const ulonglong2* nlq = reinterpret_cast<const ulonglong2*>(ost + kBTile + 512);
      if (!__all_sync(0xFFFFFFFFu, wait_bar(bar(kKBarST), uint32_t(i) & 1u, ctl, p.status,
                                            p.timeout_ns) &&
                                       wait_bar(bar(kKBarOF + i % kKOSlots),
                                                uint32_t(i / kKOSlots) & 1u, ctl, p.status,
                                                p.timeout_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[64], dp[64];
      tmem_ld32(tR + 32 * half, s);
      tmem_ld32(tR + 64 + 32 * half, s + 32);
      tmem_wait_ld();
      // Pᵀ into region(i) columns [32 half + 16 b, +16), over scores this
      // thread has read; dV += Pᵀ dO starts on its barrier
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const int cb = 64 * b + 32 * half;
        uint64_t nl2[16];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const ulonglong2 l = nlq[cb / 4 + k];
          nl2[2 * k] = l.x;
          nl2[2 * k + 1] = l.y;
        }
        float(&sb)[32] = *reinterpret_cast<float(*)[32]>(s + 32 * b);
        uint32_t pw[16];
        if (cls == SCA_TILE_FULL) p_pairs<true>(sb, 0u, c2, nl2, pw);
        else p_pairs<false>(sb, vis[b], c2, nl2, pw);
        tmem_st16(tR + 32 * half + 16 * b, pw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kKBarPR));
      if (!__all_sync(0xFFFFFFFFu, wait_bar(bar(kKBarDPT), uint32_t(i) & 1u, ctl, p.status,
                                            p.timeout_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_ld32(tD + 32 * half, dp);
      tmem_ld32(tD + 64 + 32 * half, dp + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(kKBarRD));  // dPᵀ is in registers: Sᵀ of the next tile may overwrite it
      // dSᵀ into region(i) columns [64 + 32 half + 16 b, +16)
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const int cb = 64 * b + 32 * half;
        uint64_t nd2[16];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const ulonglong2 d = ndq[cb / 4 + k];
          nd2[2 * k] = d.x;
          nd2[2 * k + 1] = d.y;
        }
        const float(&pb)[32] = *reinterpret_cast<const float(*)[32]>(s + 32 * b);
        const float(&dpb)[32] = *reinterpret_cast<const float(*)[32]>(dp + 32 * b);
        uint32_t dsw[16];
        ds_from_p(pb, dpb, nd2, dsw);
        tmem_st16(tR + 64 + 32 * half + 16 * b, dsw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kKBarDS));
    }
    // epilogue: dV and dK rows (this half)
    if (ok) ok = wait_bar(bar(kKBarDone), 0, ctl, p.status, p.timeout_ns);
    if (__all_sync(0xFFFFFFFFu, ok)) {
      tc_fence_after();
      float gv[64], gk[64];
      if (n > 0) {
        tmem_ld32(tDV + lane_base + c0, gv);
        tmem_ld32(tDV + lane_base + c0 + 32, gv + 32);
        tmem_ld32(tDK + lane_base + c0, gk);
        tmem_ld32(tDK + lane_base + c0 + 32, gk + 32);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) gv[c] = gk[c] = 0.f;
      }
      if (key < p.n) {
        const int64_t off = (int64_t(key) * p.heads + head) * 128 + c0;
        uint4* ov = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dv) + off);
        uint4* ok4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dk) + off);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          ov[c] = make_uint4(pack_bf16(gv[8 * c], gv[8 * c + 1]), pack_bf16(gv[8 * c + 2], gv[8 * c + 3]),
                             pack_bf16(gv[8 * c + 4], gv[8 * c + 5]), pack_bf16(gv[8 * c + 6], gv[8 * c + 7]));
          ok4[c] = make_uint4(pack_bf16(gk[8 * c] * p.scale, gk[8 * c + 1] * p.scale),
                              pack_bf16(gk[8 * c + 2] * p.scale, gk[8 * c + 3] * p.scale),
                              pack_bf16(gk[8 * c + 4] * p.scale, gk[8 * c + 5] * p.scale),
                              pack_bf16(gk[8 * c + 6] * p.scale, gk[8 * c + 7] * p.scale));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

cudaError_t launch_backward(const BwdMaps& maps, const BwdArgs& args, cudaStream_t stream) {
  // devices whose kernel attributes are set (a set bit; set at most once
  // per device, safely from several host threads)
  static std::atomic<uint32_t> configured_mask{0u};
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 31 || !(configured_mask.load() & (1u << dev))) {
    e = cudaFuncSetAttribute(bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kQSmem));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(kKSmem));
    if (e != cudaSuccess) return e;
    if (dev < 31) configured_mask.fetch_or(1u << dev);
  }
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t rows = int64_t(args.n_pad) * args.heads;
  int64_t blocks = (rows + 7) / 8;
  blocks = blocks < int64_t(sms) * 16 ? blocks : int64_t(sms) * 16;
  bwd_prep_kernel<<<unsigned(blocks), 256, 0, stream>>>(args);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_dq_kernel<<<unsigned(args.n_pairs * 2 * args.heads), kBThreads, kQSmem, stream>>>(
      maps.q, maps.k, maps.v, maps.d_o, args);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_dkdv_kernel<<<unsigned(args.n_q_tiles * args.heads), kBThreads, kKSmem, stream>>>(
      maps.q, maps.k, maps.v, maps.d_o, maps.dl, args);
  return cudaGetLastError();
}

}  // namespace sca
