// Camera cross-attention of libsca for NVIDIA B200 (sm_100a): the attention
// core of Eq. 3 of [picx.dev summary, Methodology › Model Architecture,
// Camera-Trajectory Conditioning], V~ = V + CrossAttn(V, C), on projected
// inputs: the visual queries of one segment attend to that segment's camera
// tokens (one per latent frame, [onedev.kr review, "어떻게 쓰나"]) and the
// result is added to a residual:
//
//   out_i = x_i + sum_f softmax_f(scale * <q_i, k_f>) v_f,  f seen by query i.
//
// Per query row and head the call moves 768 bytes through HBM (q and x in,
// out back) for two small products (128 x n_cam and n_cam x 128), so it is
// bound by HBM. The kernel keeps the memory system busy and spends as few
// instructions per row as it can:
//
// * Persistent: one CTA per SM takes a contiguous range of the (head, 128-row
//   tile) work items.
// * A producer thread streams every tile's q (two 64-column halves of 128
//   rows, 128-byte swizzle) with TMA tensor copies into a ring of stages, and
//   the camera K and V of each head once per run of tiles of that head; the
//   tiles' x come the same way into a ring of their own (see the store
//   thread), so neither stream waits behind the other.
// * One thread issues the products on the 5th-generation tensor cores:
//   S = Q Kᵀ (M = 128, N = n_cam rounded up to 16, K = 128) into tensor
//   memory, then O = P V (M = 128, N = 128, K = n_cam rounded up to 16) with
//   P read from tensor memory, where the softmax left it over S.
// * Two warpgroups take alternate tiles, one thread per row: the masked
//   softmax of the row's S (fp32; P rounded to bf16 for its product, as in
//   the main attention kernel), then x + O / l formed over x in the staged
//   tile, with packed two-lane fp32 arithmetic.
// * A store thread writes each finished tile back with a TMA tensor store and,
//   once the store has read the stage, loads the x of the tile that uses the
//   stage next. Each warpgroup has an x stage of its own (and two store
//   barriers), so that every barrier's phases are waited for in order by the
//   one warpgroup that uses it: with one ring shared by both, a warpgroup
//   could wait on a stage's next phase before the other one's had completed,
//   and a parity wait would take the incomplete phase for the awaited one.
// * Launched as a programmatic dependent of the work before it on the stream:
//   the CTAs allocate tensor memory and set up their barriers while that work
//   finishes, then wait for it (griddepcontrol.wait) before any global memory
//   access; each call lets the next one launch early in the same way.
// * Every wait is bounded: a wait that runs out sets SCA_ERR_DEVICE_TIMEOUT in
//   the status word, every role lets its own copies and products in flight
//   complete, and the CTA frees its tensor memory and exits.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "sca_camera.h"
#include "sca_ptx.cuh"

namespace sca {

namespace {

constexpr int kThreads = 352;  // producer, MMA, two epilogue warpgroups, store
constexpr int kProducerWarp = 0, kMmaWarp = 1, kEpiWarp0 = 2, kStoreWarp = 10;
constexpr int kHalf = 128 * 128;        // one 64-column half of a 128-row tile
constexpr int kTile = 2 * kHalf;        // a 128-row tile of q or x
template <int NF>  // camera tokens rounded up to 16
struct CamLayout {
  // x stages per epilogue warpgroup, q stages (measured: 3 q stages and one x
  // stage per warpgroup beat 2 and 2)
  static constexpr int kXPerWg = 1;
  static constexpr int kXStages = 2 * kXPerWg;
  static constexpr int kQStages = 3;
  static constexpr int kKVHalf = NF * 128;           // a 64-column half of K or V
  static constexpr int kKV = 4 * kKVHalf;            // K and V of one head
  // barriers (8 bytes each) and control words in the first 1024 bytes
  static constexpr int kBarKVFull = 0, kBarKVEmpty = 2, kBarQFull = 4,
                       kBarQEmpty = kBarQFull + kQStages, kBarXFull = kBarQEmpty + kQStages,
                       kBarS = kBarXFull + kXStages,
                       kBarP = kBarS + 2, kBarO = kBarP + 2, kBarStore = kBarO + 2,
                       kBarDrain = kBarStore + 4,
                       kNumBars = kBarDrain + 1;
  static constexpr int kOffCtl = 1000, kOffTmem = 1008;
  static constexpr int kOffQ = 1024;
  static constexpr int kOffX = kOffQ + kQStages * kTile;
  static constexpr int kOffKV = kOffX + kXStages * kTile;
  static constexpr int kBytes = kOffKV + 2 * kKV;
  static constexpr int kSmem = kBytes + 1024;        // room to align the base to 1024
  static_assert(kNumBars * 8 <= kOffCtl, "barrier area");
  static_assert(kSmem <= 227 * 1024, "shared memory of one CTA");
};

// Instruction descriptors, kind::f16: bf16 A and B, fp32 D, M = 128.
template <int N, bool kBMnMajor>
__host__ __device__ constexpr uint32_t idesc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (kBMnMajor ? (1u << 16) : 0u) |
         (uint32_t(N >> 3) << 17) | ((128u >> 4) << 24);
}

// MN-major operand with 128-byte swizzle whose two 64-element halves along N
// lie `lbo` bytes apart (8-row groups along K 1024 bytes apart).
__device__ __forceinline__ uint64_t desc_mn(uint32_t saddr, uint32_t lbo) {
  return uint64_t((saddr & 0x3FFFFu) >> 4) | (uint64_t(lbo >> 4) << 16) |
         (uint64_t(1024 >> 4) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// D (+)= A B with A and B in shared memory
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t id,
                                       uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(id), "r"(acc)
      : "memory");
}

// D (+)= A B with A in tensor memory
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t id,
                                       uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(id), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* r) {
  uint32_t* u = reinterpret_cast<uint32_t*>(r);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
        "=r"(u[7]), "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]),
        "=r"(u[14]), "=r"(u[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* u) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
      "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7])
      : "memory");
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int32_t c0,
                                             int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Camera tokens [lo, hi) seen by a query of latent frame fr (see sca.h).
__device__ __forceinline__ int2 cam_range(int fr, int n_cam, int mode) {
  if (mode == SCA_CAM_ALL) return make_int2(0, n_cam);
  if (fr < 0 || fr >= n_cam) return make_int2(0, 0);
  return mode == SCA_CAM_OWN_FRAME ? make_int2(fr, fr + 1) : make_int2(0, fr + 1);
}

template <int NF>
__global__ void __launch_bounds__(kThreads, 1)
    camera_xattn_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_out,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const CamArgs a) {
  using L = CamLayout<NF>;
  constexpr int kXS = L::kXStages, kQStages = L::kQStages, kXPerWg = L::kXPerWg;
  // tile k, the m-th tile (m = k / 2) of warpgroup k % 2: its x stage, the
  // use of that stage it is, and its store barrier
  auto x_stage = [&](int k) { return (k & 1) * kXPerWg + (k >> 1) % kXPerWg; };
  auto x_use = [&](int k) { return (k >> 1) / kXPerWg; };
  auto store_bar = [&](int k) { return L::kBarStore + 2 * (k & 1) + ((k >> 1) & 1); };
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* const smem = smem_raw + (sbase - raw);
  volatile Ctl* const ctl = reinterpret_cast<Ctl*>(smem + L::kOffCtl);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffTmem);
  auto bar = [&](int i) { return sbase + uint32_t(i) * 8u; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int H = a.heads;
  const int n_tiles = (a.n_q + 127) / 128;
  const int64_t total = int64_t(n_tiles) * H;
  const int64_t w0 = total * blockIdx.x / gridDim.x, w1 = total * (blockIdx.x + 1) / gridDim.x;
  const int n = int(w1 - w0);  // tiles of this CTA, head-major
  auto head_of = [&](int k) { return int((w0 + k) / n_tiles); };
  auto row0_of = [&](int k) { return int((w0 + k) % n_tiles) * 128; };

  if (threadIdx.x == 0) {
    ctl->abort = 0;
    for (int i = 0; i < L::kNumBars; ++i) {
      const bool wg = (i >= L::kBarP && i < L::kBarO) || (i >= L::kBarStore && i < L::kBarDrain);
      mbar_init(bar(i), wg ? 128 : 1);
    }
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
  // the next launch on the stream may be scheduled now; this one reads and
  // writes global memory only once the work before it has completed
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int run = -1, h_prev = -1, k = 0;
      bool ok = true;
      for (; k < n; ++k) {
        const int h = head_of(k), r0 = row0_of(k);
        if (h != h_prev) {  // a new run of tiles of head h: its camera K and V
          if (run >= 1)
            ok = wait_bar(bar(L::kBarKVEmpty + ((run + 1) & 1)), uint32_t(((run + 1) >> 1) - 1) & 1u,
                          ctl, a.status, a.timeout_ns);
          if (!ok) break;
          ++run;
          h_prev = h;
          const int e = run & 1;
          const uint32_t dst = sbase + L::kOffKV + uint32_t(e) * L::kKV;
          mbar_expect_tx(bar(L::kBarKVFull + e), uint32_t(L::kKV));
          tma_load_3d(dst, &tm_k, bar(L::kBarKVFull + e), 0, h, 0);
          tma_load_3d(dst + L::kKVHalf, &tm_k, bar(L::kBarKVFull + e), 64, h, 0);
          tma_load_3d(dst + 2 * L::kKVHalf, &tm_v, bar(L::kBarKVFull + e), 0, h, 0);
          tma_load_3d(dst + 3 * L::kKVHalf, &tm_v, bar(L::kBarKVFull + e), 64, h, 0);
        }
        const int sq = k % kQStages;
        if (k >= kQStages)
          ok = wait_bar(bar(L::kBarQEmpty + sq), uint32_t(k / kQStages - 1) & 1u, ctl, a.status,
                        a.timeout_ns);
        if (!ok) break;
        const uint32_t dq = sbase + L::kOffQ + uint32_t(sq) * kTile;
        mbar_expect_tx(bar(L::kBarQFull + sq), uint32_t(kTile));
        tma_load_3d(dq, &tm_q, bar(L::kBarQFull + sq), 0, h, r0);
        tma_load_3d(dq + kHalf, &tm_q, bar(L::kBarQFull + sq), 64, h, r0);
      }
      // Drain (after a normal end every phase has long completed): the latest
      // copy armed into each stage lands before the CTA can exit. Tiles
      // 0 .. k-1 have their q armed; runs 0 .. run their K and V.
      for (int i = k - kQStages < 0 ? 0 : k - kQStages; i < k; ++i)
        wait_drain(bar(L::kBarQFull + i % kQStages), uint32_t(i / kQStages) & 1u);
      for (int rr = run - 1 < 0 ? 0 : run - 1; rr <= run; ++rr)
        wait_drain(bar(L::kBarKVFull + (rr & 1)), uint32_t(rr >> 1) & 1u);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc<NF, false>(), kIdO = idesc<128, true>();
      bool ok = true;
      int run = -1, h_prev = -1;
      // O_j = P_j V for tile i of run ri; the run's K/V entry is released
      // after the last tile of the run. (Warpgroup j writes P of tile i only
      // after it has read O of tile i - 2, so O_j is free once P_j is ready.)
      auto pv = [&](int i, int ri, bool last_of_run) {
        const int j = i & 1;
        ok = wait_bar(bar(L::kBarP + j), uint32_t(i >> 1) & 1u, ctl, a.status, a.timeout_ns);
        if (!ok) return;
        tc_fence_after();
        const uint32_t tS = tmem + uint32_t(j) * 64, tO = tmem + 128 + uint32_t(j) * 128;
        const uint32_t sV = sbase + L::kOffKV + uint32_t(ri & 1) * L::kKV + 2 * L::kKVHalf;
#pragma unroll
        for (int kk = 0; kk < NF / 16; ++kk)
          mma_ts(tO, tS + uint32_t(kk) * 8, desc_mn(sV + uint32_t(kk) * 2048, L::kKVHalf), kIdO,
                 kk > 0 ? 1u : 0u);
        mma_commit(bar(L::kBarO + j));
        if (last_of_run) mma_commit(bar(L::kBarKVEmpty + (ri & 1)));
      };
      int run_prev = 0;
      for (int k = 0; k < n && ok; ++k) {
        const int h = head_of(k);
        if (h != h_prev) {
          ++run;
          h_prev = h;
          ok = wait_bar(bar(L::kBarKVFull + (run & 1)), uint32_t(run >> 1) & 1u, ctl, a.status,
                        a.timeout_ns);
          if (!ok) break;
        }
        const int sq = k % kQStages, j = k & 1;
        ok = wait_bar(bar(L::kBarQFull + sq), uint32_t(k / kQStages) & 1u, ctl, a.status,
                      a.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sQ = sbase + L::kOffQ + uint32_t(sq) * kTile;
        const uint32_t sK = sbase + L::kOffKV + uint32_t(run & 1) * L::kKV;
        const uint32_t tS = tmem + uint32_t(j) * 64;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = uint32_t(ks & 3) * 32;
          mma_ss(tS, desc_kmajor(sQ + uint32_t(ks >> 2) * kHalf + off),
                 desc_kmajor(sK + uint32_t(ks >> 2) * L::kKVHalf + off), kIdS, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar(L::kBarQEmpty + sq));
        mma_commit(bar(L::kBarS + j));
        if (k >= 1) pv(k - 1, run_prev, h != head_of(k - 1));
        run_prev = run;
      }
      if (ok && n > 0) pv(n - 1, run_prev, true);
      // every product has finished before this thread leaves (also on abort)
      mma_commit(bar(L::kBarDrain));
      wait_drain(bar(L::kBarDrain), 0);
    }
    __syncwarp();
  } else if (warp == kStoreWarp) {
    // ------------------------------------------------------------ store
    if (lane == 0) {
      auto load_x = [&](int k) {
        const int sx = x_stage(k);
        const uint32_t dx = sbase + L::kOffX + uint32_t(sx) * kTile;
        mbar_expect_tx(bar(L::kBarXFull + sx), uint32_t(kTile));
        tma_load_3d(dx, &tm_x, bar(L::kBarXFull + sx), 0, head_of(k), row0_of(k));
        tma_load_3d(dx + kHalf, &tm_x, bar(L::kBarXFull + sx), 64, head_of(k), row0_of(k));
      };
      // the next tile in tile k's stage is k + kXS (kXPerWg tiles of the same
      // warpgroup later); x loads go out in tile order
      int loaded = 0;  // x of tiles 0 .. loaded-1 armed
      for (; loaded < n && loaded < kXS; ++loaded) load_x(loaded);
      bool stored = false;
      for (int k = 0; k < n; ++k) {
        if (!wait_bar(bar(store_bar(k)), uint32_t(k >> 2) & 1u, ctl, a.status, a.timeout_ns))
          break;
        const uint32_t src = sbase + L::kOffX + uint32_t(x_stage(k)) * kTile;
        tma_store_3d(&tm_out, src, 0, head_of(k), row0_of(k));
        tma_store_3d(&tm_out, src + kHalf, 64, head_of(k), row0_of(k));
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        stored = true;
        // once the copy has read the stage, it takes the x of tile k + kXS
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        if (loaded < n) load_x(loaded++);
      }
      // the output writes are complete, and every x copy armed has landed,
      // before the CTA exits (the last kXS tiles armed are in distinct stages)
      if (stored) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
      for (int i = loaded - kXS < 0 ? 0 : loaded - kXS; i < loaded; ++i)
        wait_drain(bar(L::kBarXFull + x_stage(i)), uint32_t(x_use(i)) & 1u);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int wg = (warp - kEpiWarp0) >> 2;   // tiles k with k % 2 == wg
    const int wq = warp & 3;                  // TMEM lane quadrant of this warp
    const int r = wq * 32 + lane;             // row in the tile
    const uint32_t lane_base = tmem + (uint32_t(wq * 32) << 16);
    const uint32_t tS = lane_base + uint32_t(wg) * 64;
    const uint32_t tO = lane_base + 128 + uint32_t(wg) * 128;
    const bool frames = a.mode != SCA_CAM_ALL;
    const uint64_t scale2 = f2(a.scale_log2, a.scale_log2);
    bool ok = true;
    for (int k = wg; k < n; k += 2) {
      const int m = k >> 1;
      const int row0 = row0_of(k);
      int fr = -1;
      if (frames && row0 + r < a.n_q) fr = __ldg(a.q_frame + row0 + r);
      const int2 rg = cam_range(fr, a.n_cam, a.mode);
      const uint32_t span = uint32_t(rg.y - rg.x);

      ok = wait_bar(bar(L::kBarS + wg), uint32_t(m) & 1u, ctl, a.status, a.timeout_ns);
      if (!__all_sync(0xFFFFFFFFu, ok)) {  // keep the warp's collective TMEM ops uniform
        ok = false;
        break;
      }
      tc_fence_after();
      float s[NF];
#pragma unroll
      for (int c = 0; c < NF / 16; ++c) tmem_ld16(tS + uint32_t(c) * 16, s + 16 * c);
      tmem_wait_ld();
      // scaled scores, the ones this row does not see at -inf; the row max
      // in four independent chains
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int f = 0; f < NF; f += 2) {
        unf2(mul2(f2(s[f], s[f + 1]), scale2), s[f], s[f + 1]);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          s[f + e] = uint32_t(f + e - rg.x) < span ? s[f + e] : -INFINITY;
          mx4[(f + e) & 3] = fmaxf(mx4[(f + e) & 3], s[f + e]);
        }
      }
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      const float nm = mx == -INFINITY ? 0.f : -mx;
      const uint64_t negm2 = f2(nm, nm);
      uint64_t acc2[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
      uint32_t pk[NF / 2];
#pragma unroll
      for (int f = 0; f < NF; f += 2) {
        float t0, t1;
        unf2(add2(f2(s[f], s[f + 1]), negm2), t0, t1);
        const float p0 = ex2(t0), p1 = ex2(t1);
        acc2[(f >> 1) & 1] = add2(acc2[(f >> 1) & 1], f2(p0, p1));
        pk[f / 2] = pack_bf16(p0, p1);
      }
#pragma unroll
      for (int c = 0; c < NF / 16; ++c) tmem_st8(tS + uint32_t(c) * 8, pk + 8 * c);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(L::kBarP + wg));
      float la, lb, lc, ld;
      unf2(acc2[0], la, lb);
      unf2(acc2[1], lc, ld);
      const float l = (la + lb) + (lc + ld);
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const uint64_t inv2 = f2(inv, inv);

      // x of the row from the staged tile (it has usually landed long before
      // O): dims 8 q .. 8 q + 7 are the 16-byte chunk q & 7 of half q >> 3,
      // swizzled by r & 7
      const int sx = x_stage(k);
      ok = wait_bar(bar(L::kBarXFull + sx), uint32_t(x_use(k)) & 1u, ctl, a.status, a.timeout_ns);
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        ok = false;
        break;
      }
      uint8_t* const xrow = smem + L::kOffX + sx * kTile + r * 128;
      const uint32_t sw = uint32_t(r & 7);
      uint4 xv[16];
#pragma unroll
      for (int q = 0; q < 16; ++q)
        xv[q] = *reinterpret_cast<const uint4*>(xrow + (q >> 3) * kHalf + ((uint32_t(q & 7) ^ sw) << 4));

      ok = wait_bar(bar(L::kBarO + wg), uint32_t(m) & 1u, ctl, a.status, a.timeout_ns);
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // x + O / l over x in the stage, 64 dims at a time
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float o[64];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld16(tO + uint32_t(hf * 64 + c * 16), o + 16 * c);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint4 xq = xv[hf * 8 + q];
          const uint32_t xw[4] = {xq.x, xq.y, xq.z, xq.w};
          uint32_t ow[4];
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            float y0, y1;
            unf2(fma2(f2(o[8 * q + 2 * w], o[8 * q + 2 * w + 1]), inv2,
                      f2(__uint_as_float(xw[w] << 16), __uint_as_float(xw[w] & 0xFFFF0000u))),
                 y0, y1);
            ow[w] = pack_bf16(y0, y1);
          }
          *reinterpret_cast<uint4*>(xrow + hf * kHalf + ((uint32_t(q) ^ sw) << 4)) =
              make_uint4(ow[0], ow[1], ow[2], ow[3]);
        }
      }
      // the row is written: the store thread sends the tile once all 128 are
      fence_proxy_async_smem();
      mbar_arrive(bar(store_bar(k)));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

template <int NF>
cudaError_t launch_nf(const CamMaps& m, const CamArgs& a, cudaStream_t stream, int dev, int sms) {
  // devices whose kernel attributes are set (a set bit; set at most once
  // per device, safely from several host threads)
  static std::atomic<uint32_t> configured_mask{0u};
  constexpr int smem = CamLayout<NF>::kSmem;
  if (dev >= 31 || !(configured_mask.load() & (1u << dev))) {
    cudaError_t e = cudaFuncSetAttribute(camera_xattn_kernel<NF>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (dev < 31) configured_mask.fetch_or(1u << dev);
  }
  const int64_t total = int64_t((a.n_q + 127) / 128) * a.heads;
  const int grid = int(total < sms ? total : sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, camera_xattn_kernel<NF>, m.q, m.x, m.out, m.k, m.v, a);
}

// SM count of each device, read once (0: not read yet)
std::atomic<int> g_sms[32];

}  // namespace

cudaError_t launch_camera_xattn(const CamMaps& maps, const CamArgs& a, cudaStream_t stream) {
  if (a.n_q == 0) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int sms = dev < 32 ? g_sms[dev].load() : 0;
  if (sms == 0) {
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (dev < 32) g_sms[dev].store(sms);
  }
  switch (camera_box_rows(a.n_cam)) {
    case 16: return launch_nf<16>(maps, a, stream, dev, sms);
    case 32: return launch_nf<32>(maps, a, stream, dev, sms);
    case 48: return launch_nf<48>(maps, a, stream, dev, sms);
    default: return launch_nf<64>(maps, a, stream, dev, sms);
  }
}

}  // namespace sca
