// math_check.cu -- test-only kernels that evaluate the attention kernels'
// hand-written math (sm100_ptx.cuh: the softcap's tanh forms) against fp64
// references on dense input sweeps and reduce the worst error on the device. Built and loaded by
// tests/test_gpu_math.py; not part of the library.
#include <cstdint>
#include <cuda_runtime.h>

#include "sm100_ptx.cuh"

namespace {

__device__ __forceinline__ void atomic_max_pos(float* dst, float v) {
  // non-negative floats order like their bit patterns
  atomicMax(reinterpret_cast<unsigned int*>(dst), __float_as_uint(v));
}


// |tanh_via_exp2(y) - tanh(y)| for y = +-10^(lo + i * step), plus y = 0.
__global__ void tanh_abs_error(float* worst, double lo, double step, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= n; i += gridDim.x * blockDim.x) {
    const double a = (i == n) ? 0.0 : pow(10.0, lo + step * i);
    for (int s = 0; s < 2; ++s) {
      const float y = static_cast<float>(s ? -a : a);
      const float t = fa::tanh_via_exp2(y);
      const double e = fabs(static_cast<double>(t) - tanh(static_cast<double>(y)));
      if (t != t) worst[1] = 1.0f;
      atomic_max_pos(&worst[0], static_cast<float>(e));
    }
  }
}

// |softcap_fma(x, 2 log2(e) / s, c, b) - (c tanh(x / s) + b)| for x =
// +-10^(lo + i * step) * s, and x = 0 (s, c, b as given).
__global__ void softcap_abs_error(float* worst, double lo, double step, int n, float s, float c, float b) {
  const float k = static_cast<float>(2.0 * 1.4426950408889634 / s);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= n; i += gridDim.x * blockDim.x) {
    const double a = (i == n) ? 0.0 : pow(10.0, lo + step * i) * s;
    for (int sg = 0; sg < 2; ++sg) {
      const float x = static_cast<float>(sg ? -a : a);
      const float t = fa::softcap_fma(x, k, c, b);
      const double e = fabs(static_cast<double>(t) - (c * tanh(static_cast<double>(x) / s) + b));
      if (t != t) worst[1] = 1.0f;
      atomic_max_pos(&worst[0], static_cast<float>(e));
    }
  }
}

}  // namespace

extern "C" int check_softcap(float* worst, double lo, double step, int n, float s, float c, float b,
                             cudaStream_t st) {
  softcap_abs_error<<<148 * 4, 256, 0, st>>>(worst, lo, step, n, s, c, b);
  return static_cast<int>(cudaGetLastError());
}

extern "C" int check_tanh(float* worst, double lo, double step, int n, cudaStream_t s) {
  tanh_abs_error<<<148 * 4, 256, 0, s>>>(worst, lo, step, n);
  return static_cast<int>(cudaGetLastError());
}
