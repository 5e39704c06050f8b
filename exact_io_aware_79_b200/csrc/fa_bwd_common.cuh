// fa_bwd_common.cuh -- indexing shared by the backward kernels: a sequence's
// lengths and first rows (fixed-length or packed layout) and the position of
// a (query head, query) in the LSE and D row vectors.
#pragma once

#include "fa_internal.h"

namespace fa {

// Sequence b's lengths and first rows (packed layout), or the fixed-length
// problem's; false when its offsets break the contract (the sequence is
// skipped).
__device__ __forceinline__ bool bwd_seq(const BwdParams& p, int b, int& Nq, int& Nk, long long& qrow,
                                        long long& krow) {
  if (p.cu_q == nullptr) {
    Nq = p.Nq;
    Nk = p.Nk;
    qrow = static_cast<long long>(b) * p.Nq;
    krow = static_cast<long long>(b) * p.Nk;
    return true;
  }
  const int q0 = p.cu_q[b], q1 = p.cu_q[b + 1], k0 = p.cu_k[b], k1 = p.cu_k[b + 1];
  if (q0 < 0 || q1 < q0 || q1 > p.total_q || q1 - q0 > p.Nq) return false;
  if (k0 < 0 || k1 < k0 || k1 > p.total_k || k1 - k0 > p.Nk) return false;
  Nq = q1 - q0;
  Nk = k1 - k0;
  qrow = q0;
  krow = k0;
  return true;
}

// Index of (query head h, query q of this sequence) in lse and dvec:
// [B, H, Nq] for fixed lengths, [H, total_q] packed.
__device__ __forceinline__ size_t rowvec_index(const BwdParams& p, int b, int h, long long qrow, int q) {
  return p.cu_q == nullptr ? (static_cast<size_t>(b) * p.H + h) * p.Nq + q
                           : static_cast<size_t>(h) * p.total_q + static_cast<size_t>(qrow + q);
}

// Keys j <= pos + right are the only visible ones when the result is >= 0
// (causal: right = 0; a right window w: right = w; both: min(0, w)); -1 when
// neither bound applies.
__device__ __forceinline__ int bwd_right_bound(const BwdParams& p) {
  if (p.window_right >= 0) return p.causal ? min(0, p.window_right) : p.window_right;
  return p.causal ? 0 : -1;
}

}  // namespace fa
