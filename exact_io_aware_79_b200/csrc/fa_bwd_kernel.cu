// fa_bwd_kernel.cu -- attention backward: dQ, dK, dV from Q, K, V, O, LSE, dO.
//
// The pages name the backward pass ("FlashAttention深度解析：从算法创新到产业
// 变革的全面影响", section 技术演进, version 2.4; "Flash-Attention v2.0 到 v2.7
// 更新", section v2.4) without stating it; it is the gradient of the forward
// definition, computed the IO-aware way: the forward's per-row LSE lets each
// tile of P be rebuilt from Q and K without the full matrix, so nothing of
// size N x N touches HBM. Per (b, h) with s = scale * Q K^T (softcapped,
// ALiBi-biased and masked as in the forward):
//   P = exp(s - LSE);  D_i = sum_c dO_ic O_ic  (= sum_j P_ij dP_ij)
//   dV = P^T dO;  dP = dO V^T;  dS = P o (dP - D) [o tanh' for softcap]
//   dQ = scale * dS K;  dK = scale * dS^T Q.
//
// One call runs three kernels: bwd_rowdot (D, and the zeroed fp32 dQ
// accumulator and job counters), the key-block kernel on the tensor cores
// (fa_bwd_tc_kernel.cu: dK and dV, and the dQ partials added into the
// accumulator), then bwd_dq_cast (dQ = scale * accumulator, to the input
// type). The deterministic mode (the pages' version 2.4 names a
// deterministic backward) drops the dQ partials and runs the fixed-order dQ
// pass (fa_bwd_dq_tc_kernel.cu) instead; every output then repeats bit for
// bit.
#include "fa_bwd_common.cuh"
#include "fa_internal.h"
#include "sm100_ptx.cuh"

#include <type_traits>

namespace fa {
namespace {

// D_i = sum_c dO_ic O_ic in fp32, [B, H, Nq]; the same threads zero their 8
// columns of the fp32 dQ accumulator or, in the deterministic mode, of dq
// itself (the fixed-order pass writes only the rows of valid sequences).
template <typename T, int D>
__global__ void __launch_bounds__(256) bwd_rowdot_kernel(const BwdParams p) {
  constexpr int LPR = D / 8;  // lanes per row
  const long long rows = static_cast<long long>(p.B) * p.Nq * p.H;
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) / LPR;
  const int cl = threadIdx.x % LPR;
  float acc = 0.0f;
  if (row < rows) {
    const size_t off = static_cast<size_t>(row) * D + cl * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.dout) + off);
    const uint4 o = *reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.out) + off);
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, ow[4] = {o.x, o.y, o.z, o.w};
    if (!p.deterministic) {
      float4* z = reinterpret_cast<float4*>(p.dq_acc + off);
      z[0] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      z[1] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    } else {
      const long long token = row / p.H, h = row % p.H;
      *reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.dq) + token * p.dq_tok + h * D + cl * 8) =
          make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = unpack2<T>(aw[e]), y = unpack2<T>(ow[e]);
      acc = fmaf(x.x, y.x, acc);
      acc = fmaf(x.y, y.y, acc);
    }
  }
#pragma unroll
  for (int o = LPR / 2; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (blockIdx.x == 0 && threadIdx.x == 0 && p.job_counter != nullptr) p.job_counter[0] = p.job_counter[1] = 0;
  if (row < rows && cl == 0) {
    // row = (b * Nq + i) * H + h  ->  dvec[(b * H + h) * Nq + i]
    const long long h = row % p.H, bi = row / p.H;
    const long long b = bi / p.Nq, i = bi % p.Nq;
    p.dvec[(b * p.H + h) * p.Nq + i] = acc;
  }
}

// dQ = scale * accumulator, cast to the input type; 4 elements per thread.
// The accumulator is [tokens, H, d]; dq rows are dq_tok elements apart.
template <typename T>
__global__ void __launch_bounds__(256) bwd_dq_cast_kernel(const BwdParams p, long long n4, int hd) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 a = reinterpret_cast<const float4*>(p.dq_acc)[i];
  uint2 w;
  w.x = pack2<T>(a.x * p.scale, a.y * p.scale);
  w.y = pack2<T>(a.z * p.scale, a.w * p.scale);
  const long long e = 4 * i, token = e / hd;
  *reinterpret_cast<uint2*>(reinterpret_cast<T*>(p.dq) + token * p.dq_tok + (e - token * hd)) = w;
}

template <typename T, int D>
cudaError_t launch(const BwdParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                   const CUtensorMap& tmO, const CUtensorMap& tmDQ, cudaStream_t stream) {
  // query rows x heads of q, dO, dQ: B * Nq fixed, total_q packed
  const long long rows = (p.cu_q == nullptr ? static_cast<long long>(p.B) * p.Nq : p.total_q) * p.H;
  const long long elems = rows * D;
  cudaError_t e = cudaSuccess;
  if (rows > 0) {
    const long long threads = rows * (D / 8);
    BwdParams pr = p;  // the row-dot kernel sees the packed layout as one sequence of total_q rows
    if (p.cu_q != nullptr) {
      pr.B = 1;
      pr.Nq = p.total_q;
    }
    bwd_rowdot_kernel<T, D><<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(pr);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // the key-block kernel (its job counter was zeroed by the row-dot kernel)
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  e = launch_bwd_tc(kBf16, D, p, tmQ, tmK, tmV, tmO, tmDQ, stream);
  if (e != cudaSuccess) return e;
  // the fixed-order dQ pass (its counter zeroed the same way)
  if (p.deterministic) return launch_bwd_dq_tc(kBf16, D, p, tmQ, tmK, tmV, tmO, stream);
  const long long n4 = elems / 4;
  if (n4 > 0)
    bwd_dq_cast_kernel<T><<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, stream>>>(p, n4, p.H * D);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd(bool bf16, int d, const BwdParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                       const CUtensorMap& tmV, const CUtensorMap& tmO, const CUtensorMap& tmDQ,
                       cudaStream_t stream) {
  if (bf16) return d == 128 ? launch<__nv_bfloat16, 128>(p, tmQ, tmK, tmV, tmO, tmDQ, stream)
                            : launch<__nv_bfloat16, 64>(p, tmQ, tmK, tmV, tmO, tmDQ, stream);
  return d == 128 ? launch<__half, 128>(p, tmQ, tmK, tmV, tmO, tmDQ, stream)
                  : launch<__half, 64>(p, tmQ, tmK, tmV, tmO, tmDQ, stream);
}

}  // namespace fa
