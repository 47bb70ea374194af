// noalloc.cu -- an allocation-free variant of sage_attn_fwd.
//
// Who needs it: some callers cannot call cudaMalloc at the point where they
// run attention.  Examples are a plugin inside an inference engine that has
// already reserved the device's memory for its own pool (a direct cudaMalloc
// then fails or fragments that pool), code written against a fixed memory
// budget that must not grow after start-up, and latency-critical callers that
// cannot accept cudaMalloc's implicit device synchronization.  Such callers
// also may have no allocator to hand a workspace buffer to sage_attn_fwd.
//
// How: the workspace lives in a file-scope __device__ array of a fixed size
// (SAGE_NOALLOC_SCRATCH_BYTES, in include/sage.h).  Every GPU that loads this
// library holds that array until the process exits.  Its device address is
// looked up once per device with cudaGetSymbolAddress -- in host code the
// array's name is only a host-side stand-in, never a device address -- and
// the call then runs the ordinary sage_attn_fwd on it.
#include <mutex>

#include "sage.h"
#include "sage_launch.cuh"

#define SAGE_EXPORT extern "C" __attribute__((visibility("default")))

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[SAGE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up on the
// first call for that device (with the device current).
sage_status_t scratch_for_current_device(void** ptr) {
  int dev = 0;
  if (sage_status_t st = sage::cuda_status(cudaGetDevice(&dev))) return st;
  if (dev < 0 || dev >= kMaxDevices) return SAGE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (sage_status_t st = sage::cuda_status(cudaGetSymbolAddress(&p, g_noalloc_scratch))) return st;
    if (!p) return SAGE_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return SAGE_OK;
}

}  // namespace

SAGE_EXPORT sage_status_t sage_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                                sage_dtype_t dtype, int B, int Hq, int Hkv, int S, int D,
                                                sage_layout_t layout, int is_causal, float sm_scale,
                                                sage_gran_t gran, sage_pv_t pv, sage_acc_t pv_accum, int smooth_k,
                                                void* stream) {
  const size_t need = sage_workspace_bytes(B, Hq, Hkv, S, D, pv, 0);
  if (need == 0) return SAGE_ERR_INVALID_ARG;
  if (need > SAGE_NOALLOC_SCRATCH_BYTES) return SAGE_ERR_WORKSPACE;   // problem too large for the array
  void* ws = nullptr;
  sage_status_t st = scratch_for_current_device(&ws);
  if (st != SAGE_OK) return st;
  // The array keeps the previous call's contents.  The pre-pass zeroes its own
  // accumulators; the device error word must start at zero too.
  if (sage_status_t st = sage::cuda_status(cudaMemsetAsync(ws, 0, 256, static_cast<cudaStream_t>(stream)))) return st;
  return sage_attn_fwd(q, k, v, out, dtype, B, Hq, Hkv, S, D, layout, is_causal, sm_scale, gran, pv, pv_accum,
                       smooth_k, 0, ws, SAGE_NOALLOC_SCRATCH_BYTES, stream);
}
