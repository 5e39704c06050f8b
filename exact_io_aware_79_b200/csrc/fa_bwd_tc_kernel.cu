// fa_bwd_tc_kernel.cu -- the backward pass's main kernel on the Blackwell
// tensor cores (tcgen05 products with TMEM accumulators, TMA tiles), head
// dimensions 64 and 128.
//
// It computes the gradient of the forward's definition (the pages name the
// backward pass: "FlashAttention深度解析：从算法创新到产业变革的全面影响",
// section 技术演进, version 2.4; "Flash-Attention v2.0 到 v2.7 更新", section
// v2.4). With s = scale Q K^T (softcapped, ALiBi-biased, masked as in the
// forward) and the forward's LSE:
//   P = exp(s - LSE), D_i = sum_c dO_ic O_ic,
//   dV = P^T dO, dP = dO V^T, dS = P o (dP - D) [o tanh' for softcap],
//   dK = scale dS^T Q, dQ = scale dS K.
// This kernel writes dK and dV and, unless the deterministic mode asks for a
// fixed-order dQ, adds the dQ partials into an fp32 accumulator.
//
// A job is one block of 128 keys of one (sequence, cache head). CTAs are
// persistent and claim jobs from a counter in the workspace, in groups of a
// few heads, key block first within a group (see tc_job). K and V of the job stay in
// shared memory and dK, dV accumulate in tensor memory while the CTA walks,
// 64 queries at a time, the query blocks of every query head that reads the
// cache head and sees a key of the block. Per query block g:
//   S^T  = K Q^T     M = 128 keys, N = 64 queries, K = d      A, B K-major
//   dP^T = V dO^T    the same
//   elementwise (one key row per TMEM lane): P^T = 2^(S^T scale log2 e -
//     LSE log2 e), dS^T = P^T o (dP^T - D); P^T goes back to TMEM as 16-bit
//     over the first half of its own S^T columns, dS^T to shared memory as
//     16-bit rows of 64 queries (128-byte swizzle)
//   dV  += P^T dO    M = 128 keys, N = d, K = 64 queries      A in TMEM, B = dO d-major
//   dQ^T = K^T dS^T  M = d, N = 64 queries, K = 128 keys      A = K d-major, B = dS^T query-major
//                    (d = 64: an M = 128 product whose rows 64..127 read the
//                    V tile after K and are never used)
//   dK  += dS^T Q    M = 128 keys, N = d, K = 64 queries      A = dS^T, B = Q d-major
// One shared-memory dS^T tile serves as the K-major A of dK and as the
// N-major B of dQ^T, and the K tile as the K-major A of S^T and the M-major
// A of dQ^T, so neither is transposed. dQ^T (one TMEM lane per dimension,
// one column per query) leaves through shared memory by TMA reduce-add into
// the fp32 accumulator.
//
// Warps: 0-7 elementwise (warp w reads TMEM lanes 32 (w % 4) .. + 31, the
// queries 32 (w / 4) .. + 31 of the block); 8-11 drain dQ^T and write dK,
// dV at the end of a job; 12 the TMA producer (and job claims); 13 the MMA
// issuer (one thread, owns TMEM).
// TMEM: dV [0, d), dK [d, 2 d); for block parity b, S^T in
// [2 d + 128 b, + 64) with P^T over it, dP^T 64 columns further with dQ^T
// over it once the elementwise warps have read dP^T.
// Shared memory (d = 128): K, V (32 KB each), three Q / dO stages (16 KB
// each), two dS^T tiles (16 KB), four fp32 dQ boxes of 32 dimensions x 64
// queries (8 KB each), the row vectors of two blocks, barriers; d = 64
// halves the K, V, Q, dO and dQ parts.
// Every wait is bounded; after a timeout the CTA stops, and the dK / dV rows
// and the dQ partials of the jobs it had claimed are written as NaN.
#include "fa_bwd_common.cuh"
#include "fa_internal.h"
#include "sm100_ptx.cuh"

#include <type_traits>

namespace fa {
namespace {

constexpr int kKeys = 128;  // keys per job
constexpr int kQb = 64;     // queries per block
constexpr int kStages = 3;  // Q / dO stages
constexpr int kRing = 4;    // per-block barrier rings
constexpr int kEwWarps = 8;
constexpr int kDrainWarp0 = 8;
constexpr int kProdWarp = 12;
constexpr int kMmaWarp = 13;
constexpr int kThreads = 14 * 32;
constexpr int kJobUsers = 1 + kEwWarps + 4;  // MMA thread, elementwise warps, drain warps
constexpr uint32_t kTmemCols = 512;
constexpr int kTileS = kKeys * kQb * 2;  // 16 KB: 128 rows of 128 bytes
constexpr int kDsBufs = 2;  // dS^T tiles
// a block's Q / dO stage and dS^T tile are freed by the same blk_done phase,
// which the producer has already seen for block g - kStages when block g
// is loaded
static_assert(kDsBufs <= kStages && kStages < kRing, "stage and dS^T reuse outrun the barrier ring");
constexpr int kBarBytes = 512;

// Layout for head dimension D (64 or 128).
template <int D>
struct TcCfg {
  static constexpr int kTileKV = kKeys * D * 2;  // K or V: D / 64 chunks of 16 KB (128 rows of 128 bytes)
  static constexpr int kTileQ = kQb * D * 2;     // a Q or dO stage: D / 64 chunks of 8 KB
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileKV;
  static constexpr int kOffQ = 2 * kTileKV;
  static constexpr int kOffO = kOffQ + kStages * kTileQ;
  static constexpr int kOffS = kOffO + kStages * kTileQ;
  static constexpr int kOffDQ = kOffS + kDsBufs * kTileS;  // D / 32 fp32 dQ boxes of 32 dimensions x 64 queries
  static constexpr int kOffRow = kOffDQ + (D / 32) * 8192;
  static constexpr int kOffBar = kOffRow + 2 * 2 * kQb * 4;
  static constexpr int kSmem = kOffBar + kBarBytes + 1024;  // + slack to align to 1 KB
  // TMEM: dV [0, D), dK [D, 2 D), then per block parity b S^T at 2 D + 128 b
  // and dP^T (later dQ^T) 64 columns further
  static constexpr uint32_t kColDV = 0, kColDK = D, kColR = 2 * D;
  // dQ^T has D rows (TMEM lanes); the drain warps holding them
  static constexpr int kDqWarps = D / 32;
  static_assert(kSmem <= 232448, "shared memory budget exceeded");
  static_assert(kColR + 256 <= 512, "TMEM budget exceeded");
};

struct TcBars {
  uint64_t kv_full;
  uint64_t q_full[kStages];
  uint64_t s_ready[kRing];   // S^T, dP^T of block g complete
  uint64_t p_ready[kRing];   // P^T in TMEM, dS^T in shared memory (elementwise warps)
  uint64_t p_free[kRing];    // dV (and dQ^T) of block g complete: its S^T columns are free, dQ^T is ready
  uint64_t dq_free[kRing];   // dQ^T of block g read out of TMEM (drain warps)
  uint64_t blk_done[kRing];  // every product of block g complete: its Q / dO stage and dS^T tile are free
  uint64_t acc_ready;        // dK, dV of the job complete (one phase per job with blocks)
  uint64_t acc_free;         // dK, dV of the previous job read out (drain warps)
  uint64_t rv_ready[2];      // row vectors of the block in slot b written (fetching warps)
  uint64_t mma_idle;
  uint64_t job_full[kJobRing];
  uint64_t job_empty[kJobRing];
  int job_id[kJobRing];
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(TcBars) <= kBarBytes, "barrier block exceeds its reserve");

// One job: key block kb of (sequence b, cache head hk), with the query
// blocks (of kQb queries) that can see one of its keys.
struct TcJob {
  int b, hk, k0, Nq, Nk, off, qb_lo, n_qb;
  int n;  // query blocks over all heads of the group; 0: none (zero dK, dV); -1: no key here
  int tb, tq0, tk0;
  long long qrow, krow;
};

// Jobs are numbered in groups of up to kHeadGroup (sequence, cache head)
// pairs, key block first within a group: the CTAs running at one time work
// on the key blocks of a few heads, so the Q / dO tiles and dQ rows those
// heads share stay in L2, and the longest jobs of a group (under a causal
// mask, its first key blocks) come first.
constexpr int kHeadGroup = 8;

__device__ __forceinline__ void tc_job(const BwdParams& p, int n_kb, int j, TcJob& J) {
  const int BH = p.B * p.H_kv;
  const int grp = j / (n_kb * kHeadGroup);
  const int rem = j - grp * n_kb * kHeadGroup;
  const int gs = min(kHeadGroup, BH - grp * kHeadGroup);
  const int kb = rem / gs, bh = grp * kHeadGroup + rem % gs;
  J.b = bh / p.H_kv;
  J.hk = bh % p.H_kv;
  J.k0 = kb * kKeys;
  J.n = -1;
  J.qb_lo = J.n_qb = 0;
  if (!bwd_seq(p, J.b, J.Nq, J.Nk, J.qrow, J.krow) || J.k0 >= J.Nk) return;
  J.tb = p.cu_q == nullptr ? J.b : 0;
  J.tq0 = p.cu_q == nullptr ? 0 : static_cast<int>(J.qrow);
  J.tk0 = p.cu_q == nullptr ? 0 : static_cast<int>(J.krow);
  J.off = J.Nk - J.Nq;  // query i sits at key position i + off
  const int k1 = min(J.k0 + kKeys, J.Nk);
  long long q_lo = 0, q_hi = J.Nq - 1;
  const int right = bwd_right_bound(p);
  if (right >= 0) q_lo = max(q_lo, static_cast<long long>(J.k0) - J.off - right);
  if (p.window_left >= 0) q_hi = min(q_hi, static_cast<long long>(k1 - 1) + p.window_left - J.off);
  if (q_lo <= q_hi) {
    J.qb_lo = static_cast<int>(q_lo / kQb);
    J.n_qb = static_cast<int>(q_hi / kQb) - J.qb_lo + 1;
  }
  J.n = (p.H / p.H_kv) * J.n_qb;
}

// Query head and first query of block u of job J.
__device__ __forceinline__ void tc_block(const BwdParams& p, const TcJob& J, int u, int& h, int& q0) {
  h = J.hk * (p.H / p.H_kv) + u / J.n_qb;
  q0 = (J.qb_lo + u % J.n_qb) * kQb;
}


// ---------------------------------------------------------------- producer

template <int D>
__device__ void tc_producer(const BwdParams& p, const CUtensorMap* tmQ, const CUtensorMap* tmK,
                            const CUtensorMap* tmV, const CUtensorMap* tmO, uint8_t* smem, TcBars* bars,
                            int n_kb, int total_jobs) {
  using C = TcCfg<D>;
  volatile int* abort = &bars->abort;
  const uint64_t pol = l2_policy_evict_last();
  auto load_q = [&](int gi, int h, int q0, int tq0, int tb) -> bool {
    const int st = gi % kStages;
    // the stage's previous block (gi - kStages) must be done with it
    if (gi >= kStages && !mbar_wait(&bars->blk_done[(gi - kStages) % kRing], ((gi - kStages) / kRing) & 1, abort))
      return false;
    mbar_arrive_expect_tx(&bars->q_full[st], 2 * C::kTileQ);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_4d(tmQ, &bars->q_full[st], smem + C::kOffQ + st * C::kTileQ + c * 8192, 64 * c, h, tq0 + q0, tb, pol);
      tma_load_4d(tmO, &bars->q_full[st], smem + C::kOffO + st * C::kTileQ + c * 8192, 64 * c, h, tq0 + q0, tb, pol);
    }
    return true;
  };
  bool ok = true;
  int nq = 0, a = 0;  // Q / dO stages and K / V tiles loaded so far (blocks are numbered by nq)
  for (int t = 0; ok; ++t) {
    int j;
    if (!publish_job(bars, p.job_counter, total_jobs, t, &j) || j < 0) break;
    TcJob J;
    tc_job(p, n_kb, j, J);
    if (J.n <= 0) continue;
    const int n = J.n, g0 = nq;
    // the first two query blocks, then K and V (they wait for the previous
    // job's last block), then the rest
    const int kv_at = min(n, 2);
    for (int u = 0; u <= n && ok; ++u) {
      if (u == kv_at) {
        if (g0 > 0 && !mbar_wait(&bars->blk_done[(g0 - 1) % kRing], ((g0 - 1) / kRing) & 1, abort)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&bars->kv_full, 2 * C::kTileKV);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            tma_load_4d(tmK, &bars->kv_full, smem + C::kOffK + c * 16384 + r * 8192, 64 * c, J.hk,
                        J.tk0 + J.k0 + 64 * r, J.tb, pol);
            tma_load_4d(tmV, &bars->kv_full, smem + C::kOffV + c * 16384 + r * 8192, 64 * c, J.hk,
                        J.tk0 + J.k0 + 64 * r, J.tb, pol);
          }
        }
        ++a;
      }
      if (u == n) break;
      int h, q0;
      tc_block(p, J, u, h, q0);
      ok = load_q(nq, h, q0, J.tq0, J.tb);
      if (ok) ++nq;
    }
  }
  // Every load issued must land before the CTA exits; on the normal path the
  // MMA thread consumed them all.
  for (int i = max(0, nq - kStages); i < nq; ++i) drain_wait(&bars->q_full[i % kStages], (i / kStages) & 1);
  if (a > 0) drain_wait(&bars->kv_full, (a - 1) & 1);
}

// ---------------------------------------------------------------- MMA issuer

template <typename T, int D, bool kDq>
__device__ void tc_mma(const BwdParams& p, uint8_t* smem, TcBars* bars, uint32_t tmem, int n_kb) {
  using C = TcCfg<D>;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t idesc_s = instr_desc_f16(kBf16, kKeys, kQb, false);     // S^T, dP^T
  constexpr uint32_t idesc_kv = instr_desc_f16(kBf16, kKeys, D, true);       // dV, dK
  // dQ^T always as an M = 128 product: for D = 64 its rows 64..127 come from
  // the V tile that follows K (16 KB on) and are never read
  constexpr uint32_t idesc_q = instr_desc_f16_ab(kBf16, 128, kQb, true, true);
  volatile int* abort = &bars->abort;
  const uint32_t sb = smem_addr(smem);
  // K-major descriptors step K by 32 bytes within a 128-byte row (and by a
  // whole chunk every 4 steps); the d-major / query-major ones step K by 16
  // rows of 128 bytes (2048 bytes)
  const uint64_t kdesc = smem_desc_sw128(sb + C::kOffK, 16, 1024);
  const uint64_t vdesc = smem_desc_sw128(sb + C::kOffV, 16, 1024);
  const uint64_t ktdesc = smem_desc_sw128(sb + C::kOffK, 16384, 1024);
  bool failed = false;
  int g = 0, a = 0;
  auto sdp = [&](int x) -> bool {
    const int st = x % kStages, b = x & 1;
    // S^T(x) goes over P^T(x - 2) (read by dV(x - 2)), dP^T(x) over
    // dQ^T(x - 2) (read out by the drain warps); S^T is issued as soon as it
    // may be, so the tensor pipe has it while the drain finishes
    if (!mbar_wait(&bars->q_full[st], (x / kStages) & 1, abort)) return false;
    if (x >= 2 && !mbar_wait(&bars->p_free[(x - 2) % kRing], ((x - 2) / kRing) & 1, abort)) return false;
    tc_fence_after();
    const uint64_t qd = smem_desc_sw128(sb + C::kOffQ + st * C::kTileQ, 16, 1024);
    const uint64_t od = smem_desc_sw128(sb + C::kOffO + st * C::kTileQ, 16, 1024);
    const uint32_t ts = tmem + C::kColR + 128 * b;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t oa = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4, ob = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
      mma_ss(ts, kdesc + oa, qd + ob, idesc_s, kk > 0 ? 1u : 0u);
    }
    if (kDq && x >= 2 && !mbar_wait(&bars->dq_free[(x - 2) % kRing], ((x - 2) / kRing) & 1, abort)) return false;
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t oa = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4, ob = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
      mma_ss(ts + 64, vdesc + oa, od + ob, idesc_s, kk > 0 ? 1u : 0u);
    }
    tc_commit(&bars->s_ready[x % kRing]);
    return true;
  };
  for (int t = 0; !failed; ++t) {
    const int j = take_job(bars, t, &failed);
    if (j < 0) break;
    TcJob J;
    tc_job(p, n_kb, j, J);
    if (J.n <= 0) continue;
    const int n = J.n;
    if (!mbar_wait(&bars->kv_full, a & 1, abort) || !sdp(g) || (n > 1 && !sdp(g + 1))) {
      failed = true;
      break;
    }
    for (int u = 0; u < n; ++u) {
      const int gi = g + u, st = gi % kStages, b = gi & 1;
      if (!mbar_wait(&bars->p_ready[gi % kRing], (gi / kRing) & 1, abort) ||
          (u == 0 && a > 0 && !mbar_wait(&bars->acc_free, (a - 1) & 1, abort))) {
        failed = true;
        break;
      }
      tc_fence_after();
      const uint32_t ts = tmem + C::kColR + 128 * b;
      const uint64_t od_mn = smem_desc_sw128(sb + C::kOffO + st * C::kTileQ, 8192, 1024);
      const uint64_t qd_mn = smem_desc_sw128(sb + C::kOffQ + st * C::kTileQ, 8192, 1024);
      const uint64_t ds = smem_desc_sw128(sb + C::kOffS + (gi % kDsBufs) * kTileS, 16, 1024);
      const uint64_t ds_mn = smem_desc_sw128(sb + C::kOffS + (gi % kDsBufs) * kTileS, 8192, 1024);
      // dV += P^T dO: the 16 queries of step kk are TMEM columns 32 (kk / 2) + 8 (kk % 2) ..
#pragma unroll
      for (int kk = 0; kk < kQb / 16; ++kk)
        mma_ts(tmem + C::kColDV, ts + 32 * (kk >> 1) + 8 * (kk & 1), od_mn + ((kk * 2048) >> 4), idesc_kv,
               (u > 0 || kk > 0) ? 1u : 0u);
      if constexpr (kDq) {
        // dQ^T = K^T dS^T over the 128 keys, into the dP^T columns
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk)
          mma_ss(ts + 64, ktdesc + ((kk * 2048) >> 4), ds_mn + ((kk * 2048) >> 4), idesc_q, kk > 0 ? 1u : 0u);
      }
      // one commit point for both: the S^T columns are free (dV read P^T)
      // and dQ^T is complete (every commit point costs the tensor pipe time)
      tc_commit(&bars->p_free[gi % kRing]);
      // dK += dS^T Q
#pragma unroll
      for (int kk = 0; kk < kQb / 16; ++kk)
        mma_ss(tmem + C::kColDK, ds + ((kk * 32) >> 4), qd_mn + ((kk * 2048) >> 4), idesc_kv,
               (u > 0 || kk > 0) ? 1u : 0u);
      tc_commit(&bars->blk_done[gi % kRing]);
      // one phase per job: the drain warps wait on it instead of on the last
      // block's ring entry, whose phase they could be two phases away from
      if (u == n - 1) tc_commit(&bars->acc_ready);
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

// ---------------------------------------------------------------- elementwise

// P^T and dS^T of 8 queries (columns c0 .. c0 + 7 of this warp's 32) for
// this thread's key: s, dp the fp32 bits of S^T and dP^T; lsen = -LSE log2 e
// and dneg = -D of the 32 queries; visible columns lo..hi (masked blocks);
// dist0 = (position of query 0) - key (ALiBi). Packed pairs -> pw, dsw.
template <typename T, bool kCap, bool kAlibi, bool kMasked>
__device__ __forceinline__ void ew_math8(const BwdParams& p, int c0, const uint32_t (&s)[32],
                                         const uint32_t (&dp)[32], const float* lsen, const float* dneg,
                                         float slope2, float dist0, int lo, int hi, uint32_t (&pw)[4],
                                         uint32_t (&dsw)[4]) {
#pragma unroll
  for (int c = 0; c < 8; c += 4) {
    const float4 ln4 = *reinterpret_cast<const float4*>(lsen + c0 + c);
    const float4 dn4 = *reinterpret_cast<const float4*>(dneg + c0 + c);
    const float ln[4] = {ln4.x, ln4.y, ln4.z, ln4.w}, dn[4] = {dn4.x, dn4.y, dn4.z, dn4.w};
#pragma unroll
    for (int e = 0; e < 4; e += 2) {
      float pr[2], dv[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int cc = c0 + c + e + i;
        const float x = __uint_as_float(s[cc]);
        float l2, f = 1.0f;
        if constexpr (kCap) {
          const float th = tanh_via_exp2(x * p.cap_scale);
          l2 = fmaf(th, p.cap_log2, ln[e + i]);
          f = fmaf(-th, th, 1.0f);
        } else {
          l2 = fmaf(x, p.scale_log2, ln[e + i]);
        }
        if constexpr (kAlibi) l2 = fmaf(-slope2, fabsf(dist0 + static_cast<float>(cc)), l2);
        float pv = ex2(l2);
        if constexpr (kMasked) pv = (cc >= lo && cc <= hi) ? pv : 0.0f;
        float d = pv * (__uint_as_float(dp[cc]) + dn[e + i]);
        if constexpr (kCap) d *= f;
        pr[i] = pv;
        dv[i] = d;
      }
      pw[(c + e) >> 1] = pack2<T>(pr[0], pr[1]);
      dsw[(c + e) >> 1] = pack2<T>(dv[0], dv[1]);
    }
  }
}

// All 32 queries of this thread: P^T to TMEM (tp: this half's first S^T
// column), dS^T to its shared-memory row (drow), 8 queries at a time.
template <typename T, bool kCap, bool kAlibi, bool kMasked>
__device__ __forceinline__ void ew_block(const BwdParams& p, const uint32_t (&s)[32], const uint32_t (&dp)[32],
                                         const float* lsen, const float* dneg, float slope2, float dist0, int lo,
                                         int hi, uint32_t tp, uint8_t* drow, int half, int row) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t pw[4], dsw[4];
    ew_math8<T, kCap, kAlibi, kMasked>(p, 8 * i, s, dp, lsen, dneg, slope2, dist0, lo, hi, pw, dsw);
    tmem_st4(tp + 4 * i, pw[0], pw[1], pw[2], pw[3]);
    *reinterpret_cast<uint4*>(drow + ((((4 * half + i) ^ (row & 7))) << 4)) = make_uint4(dsw[0], dsw[1], dsw[2], dsw[3]);
  }
}

template <typename T, bool kCap, bool kAlibi>
__device__ __forceinline__ void ew_block_any(bool masked, const BwdParams& p, const uint32_t (&s)[32],
                                             const uint32_t (&dp)[32], const float* lsen, const float* dneg,
                                             float slope2, float dist0, int lo, int hi, uint32_t tp, uint8_t* drow,
                                             int half, int row) {
  if (masked)
    ew_block<T, kCap, kAlibi, true>(p, s, dp, lsen, dneg, slope2, dist0, lo, hi, tp, drow, half, row);
  else
    ew_block<T, kCap, kAlibi, false>(p, s, dp, lsen, dneg, slope2, dist0, lo, hi, tp, drow, half, row);
}

template <typename T, int D>
__device__ void tc_elementwise(const BwdParams& p, uint8_t* smem, TcBars* bars, uint32_t tmem, int n_kb, int warp,
                               int lane) {
  using C = TcCfg<D>;
  volatile int* abort = &bars->abort;
  const int quarter = warp & 3, half = warp >> 2;
  const int row = 32 * quarter + lane;
  const int et = warp * 32 + lane;  // 0..255: threads 0..127 fetch the row vectors
  const uint32_t tl = tmem + (static_cast<uint32_t>(32 * quarter) << 16);
  float* srow = reinterpret_cast<float*>(smem + C::kOffRow);  // [2][-lse log2 e x 64 | -D x 64]
  uint8_t* sds = smem + C::kOffS;
  const bool alibi = p.slopes != nullptr;
  const int right = bwd_right_bound(p);
  bool failed = false;
  int g = 0;
  for (int t = 0; !failed; ++t) {
    const int j = take_job_warp(bars, t, lane, &failed);
    if (j < 0) break;
    TcJob J;
    tc_job(p, n_kb, j, J);
    if (J.n <= 0) continue;
    const int n = J.n;
    const int key = J.k0 + row;
    // row vector entry of block u for this thread (et < 128): LSE of query
    // et (et < 64) or D of query et - 64, as loaded; the value is only
    // transformed when it is stored a block later, so the load stays in
    // flight meanwhile
    auto fetch = [&](int u) -> float {
      int h, q0;
      tc_block(p, J, u, h, q0);
      const int q = q0 + (et & (kQb - 1));
      if (et >= 2 * kQb) return 0.0f;
      if (q >= J.Nq) return et < kQb ? INFINITY : 0.0f;
      const size_t ri = rowvec_index(p, J.b, h, J.qrow, q);
      return et < kQb ? p.lse[ri] : p.dvec[ri];
    };
    float rv = fetch(0);
    for (int u = 0; u < n; ++u) {
      const int gi = g + u, b = gi & 1;
      int h, q0;
      tc_block(p, J, u, h, q0);
      bool ok = mbar_wait(&bars->s_ready[gi % kRing], (gi / kRing) & 1, abort);
      if (__any_sync(0xffffffffu, !ok)) {
        failed = true;
        break;
      }
      // Row vectors of block gi into slot b. Every elementwise warp has read
      // the slot's previous block (gi - 2) before S^T(gi) could be computed
      // (that product waited for dV(gi - 2), which waited for all of them).
      if (warp < 4) {
        srow[b * 2 * kQb + et] = et < kQb ? -rv * kLog2e : -rv;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->rv_ready[b]);
      }
      ok = mbar_wait(&bars->rv_ready[b], (gi >> 1) & 1, abort);
      if (__any_sync(0xffffffffu, !ok)) {
        failed = true;
        break;
      }
      if (u + 1 < n) rv = fetch(u + 1);
      // dS^T tile gi % kDsBufs was last read by the products of block gi - kDsBufs
      ok = gi < kDsBufs ||
           mbar_wait(&bars->blk_done[(gi - kDsBufs) % kRing], ((gi - kDsBufs) / kRing) & 1, abort);
      if (__any_sync(0xffffffffu, !ok)) {
        failed = true;
        break;
      }
      tc_fence_after();
      uint32_t s[32], dp[32];
      tmem_ld32(tl + C::kColR + 128 * b + 32 * half, s);
      tmem_ld32(tl + C::kColR + 128 * b + 64 + 32 * half, dp);
      // block-level mask decision (uniform over the CTA)
      bool full = J.k0 + kKeys <= J.Nk && q0 + kQb <= J.Nq;
      if (right >= 0) full = full && J.k0 + kKeys - 1 <= q0 + J.off + right;
      if (p.window_left >= 0) full = full && J.k0 >= q0 + kQb - 1 + J.off - p.window_left;
      // this thread's visible columns lo..hi of its 32 queries
      const int qb = q0 + 32 * half;
      int lo = 0, hi = min(31, J.Nq - qb - 1);
      if (key >= J.Nk) hi = -1;
      if (right >= 0) lo = max(lo, key - qb - J.off - right);
      if (p.window_left >= 0) hi = min(hi, key - qb - J.off + p.window_left);
      const float slope2 = alibi ? p.slopes[h] * kLog2e : 0.0f;
      const float dist0 = static_cast<float>(qb + J.off - key);
      const float* lsen = srow + b * 2 * kQb + 32 * half;
      const float* dneg = lsen + kQb;
      tmem_wait_ld();
      reg_fence(s);
      reg_fence(dp);
      const uint32_t tp = tl + C::kColR + 128 * b + 32 * half;  // P^T over this half's first S^T columns
      uint8_t* drow = sds + (gi % kDsBufs) * kTileS + row * 128;
      if (p.use_softcap) {
        if (alibi) ew_block_any<T, true, true>(!full, p, s, dp, lsen, dneg, slope2, dist0, lo, hi, tp, drow, half, row);
        else ew_block_any<T, true, false>(!full, p, s, dp, lsen, dneg, slope2, dist0, lo, hi, tp, drow, half, row);
      } else {
        if (alibi) ew_block_any<T, false, true>(!full, p, s, dp, lsen, dneg, slope2, dist0, lo, hi, tp, drow, half, row);
        else ew_block_any<T, false, false>(!full, p, s, dp, lsen, dneg, slope2, dist0, lo, hi, tp, drow, half, row);
      }
      tmem_wait_st();
      fence_proxy_async_shared();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_ready[gi % kRing]);
    }
    g += n;
  }
}

// ---------------------------------------------------------------- drain / epilogue

template <typename T>
__device__ __forceinline__ void store_row16(T* dst, const uint32_t (&r)[32], float mul, bool nan) {
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float x0 = nan ? __int_as_float(0x7fc00000) : __uint_as_float(r[2 * i]) * mul;
    const float x1 = nan ? __int_as_float(0x7fc00000) : __uint_as_float(r[2 * i + 1]) * mul;
    w[i] = pack2<T>(x0, x1);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
    reinterpret_cast<uint4*>(dst)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
}

template <typename T, int D, bool kDq>
__device__ void tc_drain(const BwdParams& p, const CUtensorMap* tmDQ, uint8_t* smem, TcBars* bars, uint32_t tmem,
                         int n_kb, int wq, int lane) {
  volatile int* abort = &bars->abort;
  using C = TcCfg<D>;
  const uint32_t tl = tmem + (static_cast<uint32_t>(32 * wq) << 16);
  float* stage = reinterpret_cast<float*>(smem + C::kOffDQ + wq * 8192);
  const bool dq_rows = wq < C::kDqWarps;  // this warp's lanes hold dQ^T rows (dimensions)
  bool failed = false;  // warp-uniform
  int g = 0, a = 0;
  for (int t = 0;; ++t) {
    bool tfail = false;
    const int j = take_job_warp(bars, t, lane, &tfail);
    if (j < 0) break;  // no job left, or none published after a failure
    TcJob J;
    tc_job(p, n_kb, j, J);
    if (J.n < 0) continue;
    const int key = J.k0 + 32 * wq + lane;
    T* dk_row = reinterpret_cast<T*>(p.dk) + static_cast<size_t>(J.krow + key) * p.dkv_tok +
                static_cast<size_t>(J.hk) * D;
    T* dv_row = reinterpret_cast<T*>(p.dv) + static_cast<size_t>(J.krow + key) * p.dkv_tok +
                static_cast<size_t>(J.hk) * D;
    if (J.n == 0) {
      // no query sees these keys: zero gradients (NaN after a failure)
      if (key < J.Nk) {
        uint32_t z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0u;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          store_row16<T>(dk_row + 32 * c, z, 1.0f, failed);
          store_row16<T>(dv_row + 32 * c, z, 1.0f, failed);
        }
      }
      continue;
    }
    const int n = J.n;
    if (kDq && dq_rows) {
      for (int u = 0; u < n; ++u) {
        const int gi = g + u;
        int h, q0;
        tc_block(p, J, u, h, q0);
        if (!failed) {
          const bool ok = mbar_wait(&bars->p_free[gi % kRing], (gi / kRing) & 1, abort);
          failed = __any_sync(0xffffffffu, !ok);
        }
        if (lane == 0) bulk_wait_read_all();  // this warp's previous reduce has read its box
        __syncwarp();
        if (!failed) tc_fence_after();
        // box row q (query), dimension 32 wq + lane: 16-byte chunk lane / 4 of
        // the 128-byte row, swizzled by q % 8; 32 queries at a time
        const uint32_t col = C::kColR + 128 * (gi & 1) + 64;
        uint32_t pa[8];  // shared address of this lane's word in rows q = 0..7 (mod 8)
#pragma unroll
        for (int k = 0; k < 8; ++k) pa[k] = smem_addr(stage) + k * 128 + ((((lane >> 2) ^ k)) << 4) + 4 * (lane & 3);
#pragma unroll 1
        for (int hq = 0; hq < 2; ++hq) {
          uint32_t r[32];
          if (!failed) {
            tmem_ld32(tl + col + 32 * hq, r);
            tmem_wait_ld();
            reg_fence(r);
          }
          if (hq == 1) {
            // dQ^T(gi) is out of TMEM: its columns may take dP^T(gi + 2)
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && !failed) mbar_arrive(&bars->dq_free[gi % kRing]);
          }
          const float nan = __int_as_float(0x7fc00000);
#pragma unroll
          for (int q = 0; q < 32; ++q)
            st_shared_f32(pa[q & 7] + (32 * hq + (q & ~7)) * 128, failed ? nan : __uint_as_float(r[q]));
        }
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_4d(tmDQ, stage, 32 * wq, h, J.tq0 + q0, J.tb);
          bulk_commit_group();
        }
      }
    }
    // dK, dV of the job
    if (!failed) {
      const bool ok = mbar_wait(&bars->acc_ready, a & 1, abort);
      failed = __any_sync(0xffffffffu, !ok);
    }
    if (!failed) tc_fence_after();
    // 32 columns at a time: dV's four pieces, then dK's (scaled)
#pragma unroll 1
    for (int c = 0; c < 2 * D / 32; ++c) {
      const bool is_k = c >= D / 32;
      const int cc = is_k ? c - D / 32 : c;
      uint32_t r[32];
      if (!failed) {
        tmem_ld32(tl + (is_k ? C::kColDK : C::kColDV) + 32 * cc, r);
        tmem_wait_ld();
        reg_fence(r);
      }
      if (key < J.Nk) store_row16<T>((is_k ? dk_row : dv_row) + 32 * cc, r, is_k ? p.scale : 1.0f, failed);
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0 && !failed) mbar_arrive(&bars->acc_free);
    g += n;
    ++a;
  }
  if (lane == 0) bulk_wait_all();
}

// ---------------------------------------------------------------- kernel

template <typename T, int D, bool kDq>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const __grid_constant__ CUtensorMap tmDQ, const BwdParams p, int n_kb, int total_jobs) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  using C = TcCfg<D>;
  TcBars* bars = reinterpret_cast<TcBars*>(smem + C::kOffBar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int i = 0; i < kStages; ++i) mbar_init(&bars->q_full[i], 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&bars->s_ready[i], 1);
      mbar_init(&bars->p_ready[i], kEwWarps);
      mbar_init(&bars->p_free[i], 1);
      mbar_init(&bars->dq_free[i], C::kDqWarps);
      mbar_init(&bars->blk_done[i], 1);
    }
    mbar_init(&bars->acc_ready, 1);
    mbar_init(&bars->acc_free, 4);
    mbar_init(&bars->rv_ready[0], 4);
    mbar_init(&bars->rv_ready[1], 4);
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
    tma_prefetch_desc(&tmDQ);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < kEwWarps) {
    tc_elementwise<T, D>(p, smem, bars, tmem, n_kb, warp, lane);
  } else if (warp < kDrainWarp0 + 4) {
    tc_drain<T, D, kDq>(p, &tmDQ, smem, bars, tmem, n_kb, warp & 3, lane);
  } else if (warp == kProdWarp) {
    if (lane == 0) tc_producer<D>(p, &tmQ, &tmK, &tmV, &tmO, smem, bars, n_kb, total_jobs);
  } else if (warp == kMmaWarp) {
    if (lane == 0) tc_mma<T, D, kDq>(p, smem, bars, tmem, n_kb);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <typename T, int D, bool kDq>
cudaError_t launch_tc(const BwdParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                      const CUtensorMap& tmO, const CUtensorMap& tmDQ, cudaStream_t stream) {
  constexpr int kSmem = TcCfg<D>::kSmem;
  auto kernel = bwd_tc_kernel<T, D, kDq>;
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
  const long long n_kb = (static_cast<long long>(p.Nk) + kKeys - 1) / kKeys;
  const long long jobs = n_kb * p.B * p.H_kv;
  if (jobs == 0) return cudaSuccess;
  if (jobs > 0x7fffffffLL) return cudaErrorInvalidValue;
  const int grid = static_cast<int>(jobs < sm_count[dev] ? jobs : sm_count[dev]);
  kernel<<<grid, kThreads, kSmem, stream>>>(tmQ, tmK, tmV, tmO, tmDQ, p, static_cast<int>(n_kb),
                                            static_cast<int>(jobs));
  return cudaGetLastError();
}

}  // namespace

template <int D>
cudaError_t launch_tc_d(bool bf16, const BwdParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                        const CUtensorMap& tmV, const CUtensorMap& tmO, const CUtensorMap& tmDQ, cudaStream_t stream) {
  const bool dq = !p.deterministic;
  if (bf16) return dq ? launch_tc<__nv_bfloat16, D, true>(p, tmQ, tmK, tmV, tmO, tmDQ, stream)
                      : launch_tc<__nv_bfloat16, D, false>(p, tmQ, tmK, tmV, tmO, tmDQ, stream);
  return dq ? launch_tc<__half, D, true>(p, tmQ, tmK, tmV, tmO, tmDQ, stream)
            : launch_tc<__half, D, false>(p, tmQ, tmK, tmV, tmO, tmDQ, stream);
}

cudaError_t launch_bwd_tc(bool bf16, int d, const BwdParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                          const CUtensorMap& tmV, const CUtensorMap& tmO, const CUtensorMap& tmDQ,
                          cudaStream_t stream) {
  return d == 128 ? launch_tc_d<128>(bf16, p, tmQ, tmK, tmV, tmO, tmDQ, stream)
                  : launch_tc_d<64>(bf16, p, tmQ, tmK, tmV, tmO, tmDQ, stream);
}

}  // namespace fa
