// fa_bwd_common.cuh -- shared by the backward kernels: a sequence's lengths
// and first rows (fixed-length or packed layout), the position of a (query
// head, query) in the LSE and D row vectors, and the job-claim ring of the
// persistent tensor-core kernels.
#pragma once

#include "fa_internal.h"
#include "sm100_ptx.cuh"

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

// ---- persistent kernels: jobs claimed from a counter, broadcast through
// a ring of job ids (Bars: job_full[kJobRing], job_empty[kJobRing] mbarriers,
// int job_id[kJobRing], int abort)

constexpr int kJobRing = 4;

// Job t of this CTA from the claim ring (every user reads every slot once
// and then frees it); -1 when the grid has no job left or the wait failed
// (then *failed is set and the slot is not freed). One thread.
template <typename Bars>
__device__ __forceinline__ int take_job(Bars* bars, int t, bool* failed) {
  const int slot = t % kJobRing;
  if (!mbar_wait(&bars->job_full[slot], (t / kJobRing) & 1, &bars->abort)) {
    *failed = true;
    return -1;
  }
  const int j = *reinterpret_cast<volatile int*>(&bars->job_id[slot]);
  mbar_arrive(&bars->job_empty[slot]);
  return j;
}

// The same for a whole warp: lane 0 takes the job, every lane gets it.
template <typename Bars>
__device__ __forceinline__ int take_job_warp(Bars* bars, int t, int lane, bool* failed) {
  bool f = false;
  int j = -1;
  if (lane == 0) j = take_job(bars, t, &f);
  j = __shfl_sync(0xffffffffu, j, 0);
  if (__shfl_sync(0xffffffffu, f ? 1 : 0, 0)) *failed = true;
  return j;
}

// Claims the next job for slot t of the ring (after its previous users
// freed it) and publishes it; -1 once the counter passes total_jobs (that
// is published too, so every user stops). False if the wait failed.
template <typename Bars>
__device__ __forceinline__ bool publish_job(Bars* bars, int* counter, int total_jobs, int t, int* job) {
  const int slot = t % kJobRing;
  if (t >= kJobRing && !mbar_wait(&bars->job_empty[slot], ((t / kJobRing) - 1) & 1, &bars->abort)) return false;
  int j = atomicAdd(counter, 1);
  if (j >= total_jobs) j = -1;
  bars->job_id[slot] = j;
  mbar_arrive(&bars->job_full[slot]);
  *job = j;
  return true;
}

// A bounded wait that ignores the abort flag (draining work in flight).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  int dummy = 0;
  mbar_wait(bar, parity, &dummy);
}

}  // namespace fa
