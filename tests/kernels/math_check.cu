// math_check.cu -- test-only kernels that evaluate the attention kernels'
// hand-written math (sm100_ptx.cuh) against fp64 references on dense input
// sweeps and reduce the worst error on the device. Built and loaded by
// tests/test_gpu_math.py; not part of the library.
#include <cstdint>
#include <cuda_runtime.h>

#include "sm100_ptx.cuh"

namespace {

__device__ __forceinline__ void atomic_max_pos(float* dst, float v) {
  // non-negative floats order like their bit patterns
  atomicMax(reinterpret_cast<unsigned int*>(dst), __float_as_uint(v));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Every fp32 f with |f| <= 1/2 (both signs): relative error of the cubic
// 2^f of ex2_poly_x2 against exp2 in fp64.
__global__ void ex2_poly_reduced(float* worst, unsigned long long n) {
  float m = 0.0f;
  const unsigned long long stride = static_cast<unsigned long long>(gridDim.x) * blockDim.x;
  for (unsigned long long i = blockIdx.x * static_cast<unsigned long long>(blockDim.x) + threadIdx.x; i < n;
       i += stride) {
    const uint32_t bits = static_cast<uint32_t>(i >> 1) | (static_cast<uint32_t>(i & 1) << 31);
    const float f = __uint_as_float(bits);
    float y0, y1;
    fa::f2_unpack(fa::ex2_poly_x2(fa::f2_pack(f, -f)), y0, y1);
    const double r0 = exp2(static_cast<double>(f)), r1 = exp2(-static_cast<double>(f));
    const double e = fmax(fabs(y0 - r0) / r0, fabs(y1 - r1) / r1);
    m = fmaxf(m, static_cast<float>(e));
  }
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) atomic_max_pos(worst, m);
}

// x = lo + i * step over the whole input range: worst[0] = largest relative
// error where 2^x is a normal float, worst[1] = largest result for
// x <= -126 (must stay at most 2^-125), worst[2] = 1 if any result was NaN,
// negative or infinite.
__global__ void ex2_poly_range(float* worst, double lo, double step, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const float x = static_cast<float>(lo + step * i);
    float y, y_inf;
    fa::f2_unpack(fa::ex2_poly_x2(fa::f2_pack(x, -INFINITY)), y, y_inf);
    if (!(y >= 0.0f) || isinf(y) || !(y_inf >= 0.0f) || y_inf > 0x1p-125f) worst[2] = 1.0f;
    const double r = exp2(static_cast<double>(x));
    if (x > -126.0f) {
      atomic_max_pos(&worst[0], static_cast<float>(fabs(y - r) / r));
    } else {
      atomic_max_pos(&worst[1], y);
    }
  }
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

extern "C" int check_ex2_poly_reduced(float* worst, cudaStream_t s) {
  // |f| <= 1/2: bit patterns 0 .. 0x3f000000, each with both signs
  const unsigned long long n = 2ull * (0x3f000000ull + 1);
  ex2_poly_reduced<<<148 * 8, 256, 0, s>>>(worst, n);
  return static_cast<int>(cudaGetLastError());
}

extern "C" int check_ex2_poly_range(float* worst, double lo, double step, int n, cudaStream_t s) {
  ex2_poly_range<<<148 * 4, 256, 0, s>>>(worst, lo, step, n);
  return static_cast<int>(cudaGetLastError());
}

extern "C" int check_tanh(float* worst, double lo, double step, int n, cudaStream_t s) {
  tanh_abs_error<<<148 * 4, 256, 0, s>>>(worst, lo, step, n);
  return static_cast<int>(cudaGetLastError());
}
