// ex2_error.cu -- test probe (not part of the library): the largest relative
// error of the GPU's approximate base-2 exponential (ex2.approx.ftz.f32), the
// instruction the attention kernel evaluates P~ with, over every float32
// argument in [lo, hi] whose exact result is a normal float32.  The oracle's
// ambiguity band assumes at most 2^-22 (two units in the last place); the
// test that builds this probe checks that assumption on the hardware.  The
// reference is the double-precision exp2 of the same argument.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// One float32 bit pattern per index: [0, npos) are the non-negative floats
// 0 .. hi, [npos, npos + nneg) the negative floats -0 .. lo.
__global__ void ex2_error_kernel(uint32_t hi_bits, uint32_t lo_abs_bits, unsigned int* worst) {
  const uint64_t npos = (uint64_t)hi_bits + 1, nneg = (uint64_t)lo_abs_bits + 1;
  const uint64_t n = npos + nneg;
  float w = 0.f;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (uint64_t)gridDim.x * blockDim.x) {
    const uint32_t bits = i < npos ? (uint32_t)i : (0x80000000u | (uint32_t)(i - npos));
    const float x = __uint_as_float(bits);
    const double ref = exp2((double)x);
    if (ref < 0x1p-126 || ref > 0x1.fffffep127) continue;     // result not a normal float32
    const double rel = fabs((double)ex2_approx(x) - ref) / ref;
    w = fmaxf(w, (float)rel * (1.0f + 0x1p-20f));              // rounded up: never under-reports
  }
  for (int o = 16; o > 0; o >>= 1) w = fmaxf(w, __shfl_xor_sync(0xffffffffu, w, o));
  if ((threadIdx.x & 31) == 0) atomicMax(worst, __float_as_uint(w));   // w >= 0: bit order = value order
}

}  // namespace

// worst: device pointer to one zeroed uint32; receives the float32 bits of
// the largest relative error.  Returns the CUDA error code of the launch.
extern "C" int ex2_max_rel_error(float lo, float hi, unsigned int* worst, void* stream) {
  if (!(lo <= 0.f && hi >= 0.f)) return (int)cudaErrorInvalidValue;
  uint32_t hb, lb;
  const float nlo = -lo;
  memcpy(&hb, &hi, 4);
  memcpy(&lb, &nlo, 4);
  ex2_error_kernel<<<148 * 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(hb, lb, worst);
  return (int)cudaGetLastError();
}
