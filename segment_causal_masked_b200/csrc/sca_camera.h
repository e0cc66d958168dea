// Launch arguments of the camera cross-attention kernel (sca_camera.cu),
// filled and validated by sca_camera_cross_attn in sca_host.cpp.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sca.h"

namespace sca {

struct CamArgs {
  const int32_t* q_frame;  // may be null for SCA_CAM_ALL
  int32_t n_q;
  int32_t n_cam;
  int32_t heads;
  int32_t mode;
  float scale_log2;        // softmax_scale · log2(e)
  int32_t* status;         // device status word (may be null)
  unsigned long long timeout_ns;  // limit of every pipeline wait
};

// Tensor maps of the call, all bf16 rows of 128 viewed as 3-D (128, heads,
// rows) with 128-byte swizzle: q, x and out with box (64, 1, 128), the camera
// K and V with box (64, 1, n_cam rounded up to 16) (rows past n_cam read as
// zeros).
struct CamMaps {
  CUtensorMap q, x, out, k, v;
};

// Rows of the camera K/V box: n_cam rounded up to a multiple of 16.
inline int camera_box_rows(int n_cam) { return (n_cam + 15) / 16 * 16; }

cudaError_t launch_camera_xattn(const CamMaps& maps, const CamArgs& a, cudaStream_t stream);

}  // namespace sca
