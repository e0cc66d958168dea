// Attention forward for callers that cannot allocate device memory.
//
// Some callers must not allocate: an inference loop with a hard latency
// budget that cannot afford the allocator (a cudaMalloc may synchronise the
// device, and may fail under memory pressure), or a runtime that embeds this
// library and whose own allocator owns all device memory, leaving nothing to
// carve a workspace from. sca_action_causal_attn_fwd allocates nothing itself
// but takes its key-split scratch from the caller. This entry point keeps
// that scratch in one fixed array that is part of the loaded library.
//
// The array lives in this file as a static __device__ object of
// SCA_STATIC_WORKSPACE_BYTES; every GPU that loads libsca holds it until the
// process exits. Host code needs its device address (the array's name is only
// a host-side stand-in): the first call on a device, with that device
// current, looks it up with cudaGetSymbolAddress and remembers it for the
// device's current context. A new context on the device (after
// cudaDeviceReset, for instance) has the array at a new address, so the
// lookup is keyed on the context's unique id and repeated when it changes.

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "sca_internal.h"

namespace sca {

// 32 MiB: the key-split partials of the 480p long-session and single-turn
// layouts at 16 heads, with and without a sliding window or a quarter of the
// video blocks, as planned for a 148-SM B200 (28 MB at most). Other SM counts
// plan other splits; a plan that does not fit runs unsplit instead.
constexpr uint64_t kStaticWorkspaceBytes = SCA_STATIC_WORKSPACE_BYTES;

static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

namespace {
constexpr int kMaxDevices = 64;

struct CachedAddress {
  void* ptr = nullptr;
  unsigned long long ctx_id = 0;  // the context the address belongs to
};

std::mutex g_ws_mutex;
CachedAddress g_ws[kMaxDevices];

typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

CtxGetIdFn ctx_get_id_fn() {
  static const CtxGetIdFn fn = []() -> CtxGetIdFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetIdFn>(p);
    return nullptr;
  }();
  return fn;
}

// Unique id of the calling thread's current context, or false when there is
// none yet (or the driver cannot tell).
bool current_ctx_id(unsigned long long* id) {
  CtxGetIdFn fn = ctx_get_id_fn();
  return fn && fn(nullptr, id) == CUDA_SUCCESS;
}
}  // namespace

// Device address of the static workspace on device `dev` (the current one),
// in the current context.
static int static_workspace(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return fail(SCA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_ws_mutex);
  unsigned long long id = 0;
  bool known = current_ctx_id(&id);
  if (!known || !g_ws[dev].ptr || g_ws[dev].ctx_id != id) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess) return check_cuda(e, "cudaGetSymbolAddress(static workspace)");
    if (!known) known = current_ctx_id(&id);  // the lookup made the primary context current
    g_ws[dev].ptr = known ? p : nullptr;      // without an id, look it up again every call
    g_ws[dev].ctx_id = id;
    *out = p;
    return SCA_OK;
  }
  *out = g_ws[dev].ptr;
  return SCA_OK;
}

}  // namespace sca

using namespace sca;

extern "C" {

int sca_action_causal_attn_fwd_static_ws(const sca_kv_cache* cache, const sca_metadata* md,
                                         int32_t heads, const void* q, const void* k_cur,
                                         const void* v_cur, void* o, float* lse,
                                         float softmax_scale, int32_t* dev_status,
                                         void* stream) {
  uint64_t need = 0;
  if (int rc = sca_attn_workspace_bytes(md, heads, &need)) return rc;
  if (need > kStaticWorkspaceBytes) {
    if (split_override() >= 2)
      return fail(SCA_ERR_CAPACITY,
                  "the forced key split needs %llu bytes of scratch; the library's static "
                  "workspace holds %llu (use sca_action_causal_attn_fwd with a caller workspace)",
                  (unsigned long long)need, (unsigned long long)kStaticWorkspaceBytes);
    // the automatic plan does not fit: run every work item whole (no scratch)
    return sca_action_causal_attn_fwd(cache, md, heads, q, k_cur, v_cur, o, lse, softmax_scale,
                                      nullptr, 0, dev_status, stream);
  }
  int dev = 0;
  if (int rc = check_cuda(cudaGetDevice(&dev), "cudaGetDevice")) return rc;
  void* ws = nullptr;
  if (int rc = static_workspace(dev, &ws)) return rc;
  return sca_action_causal_attn_fwd(cache, md, heads, q, k_cur, v_cur, o, lse, softmax_scale, ws,
                                    kStaticWorkspaceBytes, dev_status, stream);
}

}  // extern "C"
