// Camera cross-attention of libsca for NVIDIA B200 (sm_100a): the attention
// core of Eq. 3 of [picx.dev summary, Methodology › Model Architecture,
// Camera-Trajectory Conditioning], V~ = V + CrossAttn(V, C), on projected
// inputs: the visual queries of one segment attend to that segment's camera
// tokens (one per latent frame, [onedev.kr review, "어떻게 쓰나"]) and the
// result is added to a residual:
//
//   out_i = x_i + sum_f softmax_f(scale * <q_i, k_f>) v_f,  f seen by query i.
//
// The work per query row is 768 bytes of HBM traffic (q and x in, out back)
// against two small products (128 x n_cam and n_cam x 128), so the kernel is
// bound by HBM. The products run on the tensor cores with warp-level
// m16n8k16 bf16 MMAs (a 16-row tile, n_cam <= 64): on the CUDA cores the
// camera rows would have to be broadcast to every row from shared memory,
// which costs more than the HBM traffic. One CTA per (block of rows, head):
// the head's camera K (row-major) and V (transposed) sit in shared memory,
// rows padded so that the fragment loads of a warp hit 32 distinct banks;
// each warp takes 16-row tiles of that head in a grid-stride loop. S and O
// stay in fp32 registers, P is rounded to bf16 for the second product (as in
// the main attention kernel).

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "sca_camera.h"

namespace sca {

namespace {

constexpr int kCamThreads = 128;  // 4 warps
constexpr int kKStride = 136;     // bf16 per K row in shared memory (128 + 8)

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float2 unpack2_bf16(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

// D = A B + D, A 16 x 16 bf16 (row), B 16 x 8 bf16 (col), D fp32
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// camera token f seen by a query of latent frame fr (see sca.h)
__device__ __forceinline__ bool cam_visible(int f, int fr, int n_cam, int mode) {
  if (f >= n_cam) return false;
  if (mode == SCA_CAM_ALL) return true;
  if (fr < 0 || fr >= n_cam) return false;
  return mode == SCA_CAM_OWN_FRAME ? f == fr : f <= fr;
}

template <int NT>  // n_cam padded to 16 * NT / 2 ... i.e. NT = n-tiles of 8 camera tokens, even
__global__ void __launch_bounds__(kCamThreads)
    camera_xattn_kernel(const CamArgs a) {
  constexpr int kFp = 8 * NT;            // padded camera tokens (a multiple of 16)
  constexpr int kVStride = kFp + 8;      // bf16 per Vᵀ row in shared memory
  __shared__ __align__(16) __nv_bfloat16 sk[kFp * kKStride];
  __shared__ __align__(16) __nv_bfloat16 svt[128 * kVStride];
  const int h = blockIdx.y;
  const int H = a.heads;
  const __nv_bfloat16* kc = static_cast<const __nv_bfloat16*>(a.k_cam);
  const __nv_bfloat16* vc = static_cast<const __nv_bfloat16*>(a.v_cam);
  // the head's camera K (rows f) and V (transposed: rows = dims), zero-padded
  for (int idx = threadIdx.x; idx < kFp * 16; idx += kCamThreads) {
    const int f = idx >> 4, c = (idx & 15) * 8;  // 8 bf16 per 16-byte chunk
    uint4 kk = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
    if (f < a.n_cam) {
      kk = *reinterpret_cast<const uint4*>(kc + (int64_t(f) * H + h) * 128 + c);
      vv = *reinterpret_cast<const uint4*>(vc + (int64_t(f) * H + h) * 128 + c);
    }
    *reinterpret_cast<uint4*>(sk + f * kKStride + c) = kk;
    const __nv_bfloat16* ve = reinterpret_cast<const __nv_bfloat16*>(&vv);
#pragma unroll
    for (int e = 0; e < 8; ++e) svt[(c + e) * kVStride + f] = ve[e];
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;  // fragment row group and column pair
  const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* xg = static_cast<const __nv_bfloat16*>(a.x);
  __nv_bfloat16* og = static_cast<__nv_bfloat16*>(a.out);
  const int n_tiles = (a.n_q + 15) / 16;
  for (int tile = blockIdx.x * (kCamThreads / 32) + warp; tile < n_tiles;
       tile += gridDim.x * (kCamThreads / 32)) {
    const int r0 = tile * 16 + g, r1 = r0 + 8;  // the two rows this lane holds
    const bool in0 = r0 < a.n_q, in1 = r1 < a.n_q;
    const uint32_t* q0 = reinterpret_cast<const uint32_t*>(qg + (int64_t(r0) * H + h) * 128);
    const uint32_t* q1 = reinterpret_cast<const uint32_t*>(qg + (int64_t(r1) * H + h) * 128);
    // S = Q Kᵀ over the 128 dims (8 k-steps of 16)
    float s[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int w = ks * 8 + t4;  // 32-bit word of the row: dims 16 ks + 2 t4, +1
      uint32_t af[4];
      af[0] = in0 ? __ldg(q0 + w) : 0u;
      af[1] = in1 ? __ldg(q1 + w) : 0u;
      af[2] = in0 ? __ldg(q0 + w + 4) : 0u;
      af[3] = in1 ? __ldg(q1 + w + 4) : 0u;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint32_t* kr = reinterpret_cast<const uint32_t*>(sk + (nt * 8 + g) * kKStride);
        mma_16816(s[nt], af, kr[w], kr[w + 4]);
      }
    }
    // masked softmax per row (the row's values are spread over the 4 lanes
    // of a quad: camera tokens nt * 8 + 2 t4, +1)
    const int fr0 = (a.q_frame && in0) ? a.q_frame[r0] : -1;
    const int fr1 = (a.q_frame && in1) ? a.q_frame[r1] : -1;
    float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int f = nt * 8 + 2 * t4 + e;
        s[nt][e] = cam_visible(f, fr0, a.n_cam, a.mode) ? s[nt][e] * a.scale_log2 : -INFINITY;
        s[nt][2 + e] = cam_visible(f, fr1, a.n_cam, a.mode) ? s[nt][2 + e] * a.scale_log2 : -INFINITY;
        m0 = fmaxf(m0, s[nt][e]);
        m1 = fmaxf(m1, s[nt][2 + e]);
      }
    }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
      m0 = fmaxf(m0, __shfl_xor_sync(0xFFFFFFFFu, m0, off));
      m1 = fmaxf(m1, __shfl_xor_sync(0xFFFFFFFFu, m1, off));
    }
    const float nm0 = m0 == -INFINITY ? 0.f : -m0, nm1 = m1 == -INFINITY ? 0.f : -m1;
    float l0 = 0.f, l1 = 0.f;
    uint32_t pf[NT / 2][4];  // P as the A fragments of the second product
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float p00 = ex2f(s[nt][0] + nm0), p01 = ex2f(s[nt][1] + nm0);
      const float p10 = ex2f(s[nt][2] + nm1), p11 = ex2f(s[nt][3] + nm1);
      l0 += p00 + p01;
      l1 += p10 + p11;
      pf[nt >> 1][(nt & 1) * 2 + 0] = pack2_bf16(p00, p01);
      pf[nt >> 1][(nt & 1) * 2 + 1] = pack2_bf16(p10, p11);
    }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
      l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, off);
      l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, off);
    }
    const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
    // O = P V, 16 n-tiles of 8 dims; out = O / l + x
    const uint32_t* x0 = reinterpret_cast<const uint32_t*>(xg + (int64_t(r0) * H + h) * 128);
    const uint32_t* x1 = reinterpret_cast<const uint32_t*>(xg + (int64_t(r1) * H + h) * 128);
    uint32_t* o0 = reinterpret_cast<uint32_t*>(og + (int64_t(r0) * H + h) * 128);
    uint32_t* o1 = reinterpret_cast<uint32_t*>(og + (int64_t(r1) * H + h) * 128);
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
      float o[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t* vr = reinterpret_cast<const uint32_t*>(svt + (dt * 8 + g) * kVStride);
#pragma unroll
      for (int ks = 0; ks < NT / 2; ++ks) mma_16816(o, pf[ks], vr[ks * 8 + t4], vr[ks * 8 + 4 + t4]);
      const int w = dt * 4 + t4;  // 32-bit word: dims 8 dt + 2 t4, +1
      if (in0) {
        const float2 xv = unpack2_bf16(x0[w]);
        o0[w] = pack2_bf16(fmaf(o[0], inv0, xv.x), fmaf(o[1], inv0, xv.y));
      }
      if (in1) {
        const float2 xv = unpack2_bf16(x1[w]);
        o1[w] = pack2_bf16(fmaf(o[2], inv1, xv.x), fmaf(o[3], inv1, xv.y));
      }
    }
  }
}

template <int NT>
cudaError_t launch_nt(const CamArgs& a, cudaStream_t stream, int sms) {
  const int n_tiles = (a.n_q + 15) / 16;
  int bx = (n_tiles + 3) / 4;
  const int cap = (4 * sms + a.heads - 1) / a.heads;  // about 4 CTAs per SM over all heads
  bx = bx < cap ? bx : cap;
  if (bx < 1) bx = 1;
  camera_xattn_kernel<NT><<<dim3(unsigned(bx), unsigned(a.heads)), kCamThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_camera_xattn(const CamArgs& a, cudaStream_t stream) {
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (a.n_q == 0) return cudaSuccess;
  if (a.n_cam <= 16) return launch_nt<2>(a, stream, sms);
  if (a.n_cam <= 32) return launch_nt<4>(a, stream, sms);
  if (a.n_cam <= 48) return launch_nt<6>(a, stream, sms);
  return launch_nt<8>(a, stream, sms);
}

}  // namespace sca
