// Launch arguments of the camera cross-attention kernel (sca_camera.cu),
// filled and validated by sca_camera_cross_attn in sca_host.cpp.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "sca.h"

namespace sca {

struct CamArgs {
  const void* q;
  const int32_t* q_frame;  // may be null for SCA_CAM_ALL
  const void* k_cam;
  const void* v_cam;
  const void* x;
  void* out;
  int32_t n_q;
  int32_t n_cam;
  int32_t heads;
  int32_t mode;
  float scale_log2;        // softmax_scale · log2(e)
};

cudaError_t launch_camera_xattn(const CamArgs& a, cudaStream_t stream);

}  // namespace sca
