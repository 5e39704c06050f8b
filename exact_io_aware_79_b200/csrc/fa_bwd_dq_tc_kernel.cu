// fa_bwd_dq_tc_kernel.cu -- the deterministic backward's dQ pass on the
// Blackwell tensor cores, head dimensions 64 and 128.
//
// The pages name a deterministic backward ("Flash-Attention v2.0 到 v2.7
// 更新", section v2.4; "FlashAttention深度解析：从算法创新到产业变革的全面影响",
// section 技术演进): every output must repeat bit for bit. dK and dV already
// do (each key block's sums run in one CTA in a fixed order); dQ sums over
// key blocks, so instead of the key-block kernel's reductions into a shared
// accumulator this pass gives every 128-query tile of one (sequence, query
// head) to one CTA, which walks the visible key blocks in increasing order
// and accumulates
//   dQ = scale * sum_j dS_j K_j,  dS_j = P_j o (dP_j - D) [o tanh'],
//   P_j = exp(s_j - LSE), dP_j = dO V_j^T
// in tensor memory, rebuilding S_j and dP_j on the way (the price of a fixed
// order: two more products per block than the key-block kernel spends on dQ).
//
// Per 64-key block g (products on tcgen05, fp32 in TMEM):
//   S  = Q K^T     M = 128 queries, N = 64 keys, K = d        A, B K-major
//   dP = dO V^T    the same
//   elementwise (one query row per TMEM lane, two warps a row, 32 keys
//     each): dS as 16-bit over the first half of its own S columns
//   dQ += dS K     M = 128 queries, N = d, K = 64 keys        A from TMEM, B = K d-major
// S and dP take one of three 128-column TMEM buffers (the buffer of block g
// is its K/V stage, so the barrier that frees a K/V stage frees the buffer);
// dQ accumulates in columns 0..d-1 and is scaled, rounded and stored by the
// elementwise warps at the end of the job.
//
// Warps: 0-7 elementwise (warp w: TMEM lanes 32 (w % 4) .., keys 32 (w / 4)
// .. + 31 of each block) and the dQ epilogue; 8 the TMA producer (and job
// claims); 9 the MMA issuer (one thread, owns TMEM). CTAs are persistent and
// claim jobs from the second workspace counter, in groups of up to eight
// (sequence, query head) pairs, the last query tile of a head first.
// Shared memory: Q and dO tiles of two jobs (32 KB each), three stages of a
// K and a V block (16 KB each), barriers. Every wait is bounded; after a
// timeout the dQ rows of the jobs the CTA had claimed are written as NaN.
#include "fa_bwd_common.cuh"
#include "fa_internal.h"
#include "sm100_ptx.cuh"

#include <type_traits>

namespace fa {
namespace {

constexpr int kBM = 128;  // queries per job
constexpr int kBN = 64;   // keys per block
constexpr int kStages = 3;
constexpr int kRing = 4;
constexpr int kEwWarps = 8;
constexpr int kProdWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = 10 * 32;
constexpr int kJobUsers = 1 + kEwWarps;  // MMA thread, elementwise warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColDQ = 0, kColBuf = 128;  // buffer s: S at 128 + 128 s, dP at + 64
constexpr int kHeadGroup = 8;

// Shared-memory regions are sized for d = 128 (d = 64 fills half of each)
constexpr int kTileQ = kBM * 128 * 2;  // 32 KB: 64-column chunks of 16 KB
constexpr int kTileK = kBN * 128 * 2;  // 16 KB: 64-column chunks of 8 KB
constexpr int kOffQ = 0;
constexpr int kOffO = 2 * kTileQ;
constexpr int kOffK = 4 * kTileQ;
constexpr int kOffV = kOffK + kStages * kTileK;
constexpr int kOffBar = kOffV + kStages * kTileK;
constexpr int kBarBytes = 512;
constexpr int kSmem = kOffBar + kBarBytes + 1024;  // + slack to align to 1 KB

struct DqBars {
  uint64_t q_full[2];        // Q, dO of job a in buffer a % 2
  uint64_t q_free[2];        // every product of job a that reads them complete
  uint64_t kv_full[kStages];
  uint64_t kv_free[kStages];  // dQ of block g complete: K/V stage and S/dP buffer g % kStages free
  uint64_t s_ready[kRing];    // S, dP of block g complete
  uint64_t ds_ready[kRing];   // dS of block g in TMEM (elementwise warps)
  uint64_t acc_ready;         // the job's dQ complete
  uint64_t acc_free;          // the previous job's dQ read out (elementwise warps)
  uint64_t mma_idle;
  uint64_t job_full[kJobRing];
  uint64_t job_empty[kJobRing];
  int job_id[kJobRing];
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(DqBars) <= kBarBytes, "barrier block exceeds its reserve");
static_assert(kSmem <= 232448, "shared memory budget exceeded");

struct DqJob {
  int b, h, hk, q0, Nq, Nk, off, kb_lo;
  int n;  // key blocks; 0: no key visible (dQ = 0); -1: no query here
  int tb, tq0, tk0;
  long long qrow, krow;
};

// Job j: query tile qt of (sequence b, query head h), numbered in groups of
// up to kHeadGroup (b, h) pairs, last query tile first within a group.
__device__ __forceinline__ void dq_job(const BwdParams& p, int n_qt, int j, DqJob& J) {
  const int BH = p.B * p.H;
  const int grp = j / (n_qt * kHeadGroup);
  const int rem = j - grp * n_qt * kHeadGroup;
  const int gs = min(kHeadGroup, BH - grp * kHeadGroup);
  const int qt = n_qt - 1 - rem / gs, bh = grp * kHeadGroup + rem % gs;
  J.b = bh / p.H;
  J.h = bh % p.H;
  J.hk = J.h / (p.H / p.H_kv);
  J.q0 = qt * kBM;
  J.n = -1;
  J.kb_lo = 0;
  if (!bwd_seq(p, J.b, J.Nq, J.Nk, J.qrow, J.krow) || J.q0 >= J.Nq) return;
  J.tb = p.cu_q == nullptr ? J.b : 0;
  J.tq0 = p.cu_q == nullptr ? 0 : static_cast<int>(J.qrow);
  J.tk0 = p.cu_q == nullptr ? 0 : static_cast<int>(J.krow);
  J.off = J.Nk - J.Nq;  // query i sits at key position i + off
  const int qmax = min(J.q0 + kBM - 1, J.Nq - 1);
  long long k_lo = 0, k_hi = J.Nk - 1;
  const int right = bwd_right_bound(p);
  if (right >= 0) k_hi = min(k_hi, static_cast<long long>(qmax) + J.off + right);
  if (p.window_left >= 0) k_lo = max(k_lo, static_cast<long long>(J.q0) + J.off - p.window_left);
  J.n = 0;
  if (k_lo <= k_hi) {
    J.kb_lo = static_cast<int>(k_lo / kBN);
    J.n = static_cast<int>(k_hi / kBN) - J.kb_lo + 1;
  }
}

// ---------------------------------------------------------------- producer

template <int D>
__device__ void dq_producer(const BwdParams& p, const CUtensorMap* tmQ, const CUtensorMap* tmK,
                            const CUtensorMap* tmV, const CUtensorMap* tmO, uint8_t* smem, DqBars* bars,
                            int n_qt, int total_jobs) {
  volatile int* abort = &bars->abort;
  const uint64_t pol = l2_policy_evict_last();
  int a = 0, nk = 0;  // jobs (with blocks) and K/V blocks loaded
  bool ok = true;
  for (int t = 0; ok; ++t) {
    int j;
    if (!publish_job(bars, p.job_counter + 1, total_jobs, t, &j) || j < 0) break;
    DqJob J;
    dq_job(p, n_qt, j, J);
    if (J.n <= 0) continue;
    const int qb = a % 2;
    if (a >= 2 && !mbar_wait(&bars->q_free[qb], ((a - 2) / 2) & 1, abort)) break;
    mbar_arrive_expect_tx(&bars->q_full[qb], 2 * kBM * D * 2);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        tma_load_4d(tmQ, &bars->q_full[qb], smem + kOffQ + qb * kTileQ + c * 16384 + r * 8192, 64 * c, J.h,
                    J.tq0 + J.q0 + 64 * r, J.tb, pol);
        tma_load_4d(tmO, &bars->q_full[qb], smem + kOffO + qb * kTileQ + c * 16384 + r * 8192, 64 * c, J.h,
                    J.tq0 + J.q0 + 64 * r, J.tb, pol);
      }
    }
    ++a;
    for (int u = 0; u < J.n; ++u) {
      const int st = nk % kStages;
      if (nk >= kStages && !mbar_wait(&bars->kv_free[st], ((nk - kStages) / kStages) & 1, abort)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(&bars->kv_full[st], 2 * kBN * D * 2);
      const int k0 = (J.kb_lo + u) * kBN;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_load_4d(tmK, &bars->kv_full[st], smem + kOffK + st * kTileK + c * 8192, 64 * c, J.hk, J.tk0 + k0, J.tb,
                    pol);
        tma_load_4d(tmV, &bars->kv_full[st], smem + kOffV + st * kTileK + c * 8192, 64 * c, J.hk, J.tk0 + k0, J.tb,
                    pol);
      }
      ++nk;
    }
  }
  // Every load issued must land before the CTA exits.
  for (int i = max(0, a - 2); i < a; ++i) drain_wait(&bars->q_full[i % 2], (i / 2) & 1);
  for (int i = max(0, nk - kStages); i < nk; ++i) drain_wait(&bars->kv_full[i % kStages], (i / kStages) & 1);
}

// ---------------------------------------------------------------- MMA issuer

template <typename T, int D>
__device__ void dq_mma(const BwdParams& p, uint8_t* smem, DqBars* bars, uint32_t tmem, int n_qt) {
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t idesc_s = instr_desc_f16(kBf16, kBM, kBN, false);  // S, dP
  constexpr uint32_t idesc_q = instr_desc_f16(kBf16, kBM, D, true);     // dQ: B = K d-major
  volatile int* abort = &bars->abort;
  const uint32_t sb = smem_addr(smem);
  bool failed = false;
  int g = 0, a = 0;
  uint64_t qd = 0, od = 0;
  // S(x), dP(x) into buffer x % kStages (its previous block's dQ is complete:
  // the producer waited for that before loading K/V stage x % kStages)
  auto sdp = [&](int x) -> bool {
    const int st = x % kStages;
    if (!mbar_wait(&bars->kv_full[st], (x / kStages) & 1, abort)) return false;
    tc_fence_after();
    const uint64_t kd = smem_desc_sw128(sb + kOffK + st * kTileK, 16, 1024);
    const uint64_t vd = smem_desc_sw128(sb + kOffV + st * kTileK, 16, 1024);
    const uint32_t ts = tmem + kColBuf + 128 * st;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t oa = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4, ob = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
      mma_ss(ts, qd + oa, kd + ob, idesc_s, kk > 0 ? 1u : 0u);
    }
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t oa = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4, ob = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
      mma_ss(ts + 64, od + oa, vd + ob, idesc_s, kk > 0 ? 1u : 0u);
    }
    tc_commit(&bars->s_ready[x % kRing]);
    return true;
  };
  for (int t = 0; !failed; ++t) {
    const int j = take_job(bars, t, &failed);
    if (j < 0) break;
    DqJob J;
    dq_job(p, n_qt, j, J);
    if (J.n <= 0) continue;
    const int n = J.n, qb = a % 2;
    if (!mbar_wait(&bars->q_full[qb], (a / 2) & 1, abort)) {
      failed = true;
      break;
    }
    qd = smem_desc_sw128(sb + kOffQ + qb * kTileQ, 16, 1024);
    od = smem_desc_sw128(sb + kOffO + qb * kTileQ, 16, 1024);
    if (!sdp(g) || (n > 1 && !sdp(g + 1))) {
      failed = true;
      break;
    }
    for (int u = 0; u < n; ++u) {
      const int gi = g + u, st = gi % kStages;
      if (!mbar_wait(&bars->ds_ready[gi % kRing], (gi / kRing) & 1, abort) ||
          (u == 0 && a > 0 && !mbar_wait(&bars->acc_free, (a - 1) & 1, abort))) {
        failed = true;
        break;
      }
      tc_fence_after();
      // dQ += dS K: the 16 keys of step kk are TMEM columns 32 (kk / 2) + 8 (kk % 2) ..
      const uint32_t ts = tmem + kColBuf + 128 * st;
      const uint64_t kmn = smem_desc_sw128(sb + kOffK + st * kTileK, 8192, 1024);
#pragma unroll
      for (int kk = 0; kk < kBN / 16; ++kk)
        mma_ts(tmem + kColDQ, ts + 32 * (kk >> 1) + 8 * (kk & 1), kmn + ((kk * 2048) >> 4), idesc_q,
               (u > 0 || kk > 0) ? 1u : 0u);
      tc_commit(&bars->kv_free[st]);
      if (u == n - 1) {
        tc_commit(&bars->q_free[qb]);
        tc_commit(&bars->acc_ready);
      }
      if (u + 2 < n && !sdp(gi + 2)) {
        failed = true;
        break;
      }
    }
    g += n;
    ++a;
  }
  // All MMAs of this thread must be complete before TMEM is released.
  tc_commit(&bars->mma_idle);
  drain_wait(&bars->mma_idle, 0);
}

// ---------------------------------------------------------------- elementwise + epilogue

// dS of 32 keys (columns c = 0..31 of this warp's half of the block) for
// this thread's query: s, dp the fp32 bits of S and dP; lsen = -LSE log2 e
// and dneg = -D of the query; visible columns lo..hi (masked blocks);
// dist0 = (query position) - (key of column 0) (ALiBi). Packed pairs -> dsw.
template <typename T, bool kCap, bool kAlibi, bool kMasked>
__device__ __forceinline__ void dq_ds(const BwdParams& p, const uint32_t (&s)[32], const uint32_t (&dp)[32],
                                      float lsen, float dneg, float slope2, float dist0, int lo, int hi,
                                      uint32_t (&dsw)[16]) {
#pragma unroll
  for (int c = 0; c < 32; c += 2) {
    float dv[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int cc = c + i;
      const float x = __uint_as_float(s[cc]);
      float l2, f = 1.0f;
      if constexpr (kCap) {
        const float th = tanh_via_exp2(x * p.cap_scale);
        l2 = fmaf(th, p.cap_log2, lsen);
        f = fmaf(-th, th, 1.0f);
      } else {
        l2 = fmaf(x, p.scale_log2, lsen);
      }
      if constexpr (kAlibi) l2 = fmaf(-slope2, fabsf(dist0 - static_cast<float>(cc)), l2);
      float pv = ex2(l2);
      if constexpr (kMasked) pv = (cc >= lo && cc <= hi) ? pv : 0.0f;
      float d = pv * (__uint_as_float(dp[cc]) + dneg);
      if constexpr (kCap) d *= f;
      dv[i] = d;
    }
    dsw[c >> 1] = pack2<T>(dv[0], dv[1]);
  }
}

template <typename T, bool kCap, bool kAlibi>
__device__ __forceinline__ void dq_ds_any(bool masked, const BwdParams& p, const uint32_t (&s)[32],
                                          const uint32_t (&dp)[32], float lsen, float dneg, float slope2,
                                          float dist0, int lo, int hi, uint32_t (&dsw)[16]) {
  if (masked)
    dq_ds<T, kCap, kAlibi, true>(p, s, dp, lsen, dneg, slope2, dist0, lo, hi, dsw);
  else
    dq_ds<T, kCap, kAlibi, false>(p, s, dp, lsen, dneg, slope2, dist0, lo, hi, dsw);
}

// 32 columns of a dQ row (scaled, or NaN / zero) as 16-bit.
template <typename T>
__device__ __forceinline__ void store_dq32(T* dst, const uint32_t (&r)[32], float mul, int what) {
  // what: 0 = values, 1 = zeros, 2 = NaN
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float x0 = __uint_as_float(r[2 * i]) * mul, x1 = __uint_as_float(r[2 * i + 1]) * mul;
    if (what == 1) x0 = x1 = 0.0f;
    if (what == 2) x0 = x1 = __int_as_float(0x7fc00000);
    w[i] = pack2<T>(x0, x1);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
    reinterpret_cast<uint4*>(dst)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
}

template <typename T, int D>
__device__ void dq_elementwise(const BwdParams& p, DqBars* bars, uint32_t tmem, int n_qt, int warp, int lane) {
  volatile int* abort = &bars->abort;
  const int quarter = warp & 3, half = warp >> 2;
  const int row = 32 * quarter + lane;
  const uint32_t tl = tmem + (static_cast<uint32_t>(32 * quarter) << 16);
  const bool alibi = p.slopes != nullptr;
  const int right = bwd_right_bound(p);
  bool failed = false;  // warp-uniform
  int g = 0, a = 0;
  for (int t = 0;; ++t) {
    bool tfail = false;
    const int j = take_job_warp(bars, t, lane, &tfail);
    if (j < 0) break;  // no job left, or none published after a failure
    DqJob J;
    dq_job(p, n_qt, j, J);
    if (J.n < 0) continue;
    const int q = J.q0 + row;
    T* dq_row = reinterpret_cast<T*>(p.dq) + static_cast<size_t>(J.qrow + q) * p.dq_tok +
                static_cast<size_t>(J.h) * D + (D / 2) * half;
    if (J.n == 0) {
      // no key visible to the tile: dQ = 0 (NaN after a failure)
      uint32_t z[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) z[i] = 0u;
      if (q < J.Nq)
        for (int c = 0; c < D / 64; ++c) store_dq32<T>(dq_row + 32 * c, z, 1.0f, failed ? 2 : 1);
      continue;
    }
    const int n = J.n;
    const size_t ri = q < J.Nq ? rowvec_index(p, J.b, J.h, J.qrow, q) : 0;
    const float lsen = q < J.Nq ? -p.lse[ri] * kLog2e : -INFINITY;
    const float dneg = q < J.Nq ? -p.dvec[ri] : 0.0f;
    const float slope2 = alibi ? p.slopes[J.h] * kLog2e : 0.0f;
    for (int u = 0; u < n && !failed; ++u) {
      const int gi = g + u, st = gi % kStages;
      const int k0 = (J.kb_lo + u) * kBN, kbase = k0 + 32 * half;
      const bool ok = mbar_wait(&bars->s_ready[gi % kRing], (gi / kRing) & 1, abort);
      if (__any_sync(0xffffffffu, !ok)) {
        failed = true;
        break;
      }
      tc_fence_after();
      uint32_t s[32], dp[32];
      const uint32_t tb = tl + kColBuf + 128 * st + 32 * half;
      tmem_ld32(tb, s);
      tmem_ld32(tb + 64, dp);
      // block-level mask decision (uniform over the CTA)
      bool full = J.q0 + kBM <= J.Nq && k0 + kBN <= J.Nk;
      if (right >= 0) full = full && k0 + kBN - 1 <= J.q0 + J.off + right;
      if (p.window_left >= 0) full = full && k0 >= J.q0 + kBM - 1 + J.off - p.window_left;
      // this thread's visible columns lo..hi of its 32 keys
      int lo = 0, hi = min(31, J.Nk - 1 - kbase);
      if (q >= J.Nq) hi = -1;
      if (right >= 0) hi = min(hi, q + J.off + right - kbase);
      if (p.window_left >= 0) lo = max(lo, q + J.off - p.window_left - kbase);
      const float dist0 = static_cast<float>(q + J.off - kbase);
      tmem_wait_ld();
      reg_fence(s);
      reg_fence(dp);
      uint32_t dsw[16];
      if (p.use_softcap) {
        if (alibi) dq_ds_any<T, true, true>(!full, p, s, dp, lsen, dneg, slope2, dist0, lo, hi, dsw);
        else dq_ds_any<T, true, false>(!full, p, s, dp, lsen, dneg, slope2, dist0, lo, hi, dsw);
      } else {
        if (alibi) dq_ds_any<T, false, true>(!full, p, s, dp, lsen, dneg, slope2, dist0, lo, hi, dsw);
        else dq_ds_any<T, false, false>(!full, p, s, dp, lsen, dneg, slope2, dist0, lo, hi, dsw);
      }
      tmem_st16(tb, dsw);  // dS over the first half of this warp's S columns
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->ds_ready[gi % kRing]);
    }
    // the job's dQ: this warp's 32 rows, columns (d / 2) half .. + d / 2 - 1
    if (!failed) {
      const bool ok = mbar_wait(&bars->acc_ready, a & 1, abort);
      failed = __any_sync(0xffffffffu, !ok);
    }
    if (!failed) tc_fence_after();
#pragma unroll 1
    for (int c = 0; c < D / 64; ++c) {
      uint32_t r[32];
      if (!failed) {
        tmem_ld32(tl + kColDQ + (D / 2) * half + 32 * c, r);
        tmem_wait_ld();
        reg_fence(r);
      }
      if (q < J.Nq) store_dq32<T>(dq_row + 32 * c, r, p.scale, failed ? 2 : 0);
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0 && !failed) mbar_arrive(&bars->acc_free);
    g += n;
    ++a;
  }
}

// ---------------------------------------------------------------- kernel

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                     const BwdParams p, int n_qt, int total_jobs) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  DqBars* bars = reinterpret_cast<DqBars*>(smem + kOffBar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->q_full[i], 1);
      mbar_init(&bars->q_free[i], 1);
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bars->kv_full[i], 1);
      mbar_init(&bars->kv_free[i], 1);
    }
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&bars->s_ready[i], 1);
      mbar_init(&bars->ds_ready[i], kEwWarps);
    }
    mbar_init(&bars->acc_ready, 1);
    mbar_init(&bars->acc_free, kEwWarps);
    mbar_init(&bars->mma_idle, 1);
    for (int i = 0; i < kJobRing; ++i) {
      mbar_init(&bars->job_full[i], 1);
      mbar_init(&bars->job_empty[i], kJobUsers);
    }
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProdWarp && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < kEwWarps) {
    dq_elementwise<T, D>(p, bars, tmem, n_qt, warp, lane);
  } else if (warp == kProdWarp) {
    if (lane == 0) dq_producer<D>(p, &tmQ, &tmK, &tmV, &tmO, smem, bars, n_qt, total_jobs);
  } else if (warp == kMmaWarp) {
    if (lane == 0) dq_mma<T, D>(p, smem, bars, tmem, n_qt);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <typename T, int D>
cudaError_t launch_dq(const BwdParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                      const CUtensorMap& tmO, cudaStream_t stream) {
  auto kernel = bwd_dq_tc_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  static int sm_count[64];
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (sm_count[dev] == 0) {
    e = cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  const long long n_qt = (static_cast<long long>(p.Nq) + kBM - 1) / kBM;
  const long long jobs = n_qt * p.B * p.H;
  if (jobs == 0) return cudaSuccess;
  if (jobs > 0x7fffffffLL) return cudaErrorInvalidValue;
  const int grid = static_cast<int>(jobs < sm_count[dev] ? jobs : sm_count[dev]);
  kernel<<<grid, kThreads, kSmem, stream>>>(tmQ, tmK, tmV, tmO, p, static_cast<int>(n_qt), static_cast<int>(jobs));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_dq_tc(bool bf16, int d, const BwdParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                             const CUtensorMap& tmV, const CUtensorMap& tmO, cudaStream_t stream) {
  if (d == 128)
    return bf16 ? launch_dq<__nv_bfloat16, 128>(p, tmQ, tmK, tmV, tmO, stream)
                : launch_dq<__half, 128>(p, tmQ, tmK, tmV, tmO, stream);
  return bf16 ? launch_dq<__nv_bfloat16, 64>(p, tmQ, tmK, tmV, tmO, stream)
              : launch_dq<__half, 64>(p, tmQ, tmK, tmV, tmO, stream);
}

}  // namespace fa
