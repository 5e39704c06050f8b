// fa_fwd_kernel.cu -- tiled exact-attention forward for sm_100a.
//
// Method (pages: "IO感知技术革命", sections on block tiling, online softmax and
// asynchronous copy; "FlashAttention深度解析", section "重新定义注意力计算";
// masking and score modifiers from "Flash-Attention v2.0 到 v2.7 更新",
// sections v2.1, v2.3, v2.4, v2.6): Q is split into 128-row tiles that stay
// on chip; K and V stream through in 128-key tiles; each K/V tile updates a
// running row max m and row sum l and rescales the partial output, so the
// N x N scores never leave the SM.
//
// B200 mapping. One CTA owns one 128-row Q tile of one (batch, head) and
// runs six warps:
//   warps 0-3  softmax, one query row per thread (row = TMEM lane)
//   warp  4    TMA producer: the Q tile once, then K_j, V_j into a ring of
//              shared-memory slots (128-byte swizzle), mbarrier expect-tx
//   warp  5    TMEM owner and MMA issuer (one elected thread)
// Tensor memory (512 columns x 128 lanes x 32 bit):
//   cols   0..127  S buffer 0 (fp32 scores; P, 16-bit, overwrites its first
//                  64 columns and feeds the PV product straight from TMEM)
//   cols 128..255  S buffer 1
//   cols 256..383  O (fp32, d columns)
// The scores are double-buffered: for K/V tile j the MMA thread issues
//   S(j+1) = Q K_{j+1}^T into the other buffer, then (once P(j) is ready)
//   O += P(j) V_j,
// so the tensor core computes the next tile's scores while the softmax
// warps work on this one, and the step time is max(softmax, tensor core)
// rather than their sum. The softmax warps are alone on the SM's four
// sub-partitions, so each has a whole MUFU (exp2) unit. tcgen05 operations
// of one thread complete in issue order, so the product that reads P(j)
// finishes before S(j+2) overwrites the same columns.
//
// Rescaling is lazy: a row keeps its old max unless a new tile raises it by
// more than 8 (log2 units), so P stays <= 2^8 and O is rescaled only when it
// must be (after waiting for the previous PV product). The result is the
// same softmax (m cancels in O / l).
#include "fa_internal.h"
#include "sm100_ptx.cuh"

#include <cfloat>
#include <climits>
#include <type_traits>

namespace fa {
namespace {

constexpr int BM = 128;  // query rows per Q tile
constexpr int BN = 128;  // keys per K/V tile
constexpr int kThreads = 192;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kMaxSlots = 12;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;

template <int D>
struct Cfg {
  static constexpr int kChunkBytes = BM * 128;       // 128 rows x 64 elements x 2 bytes
  static constexpr int kTileBytes = BM * D * 2;      // one Q, K or V tile
  static constexpr int kSlots = (D == 128) ? 6 : 12; // K/V ring depth
  static constexpr int kSmemBytes = 1024 + (1 + kSlots) * kTileBytes + 1024;
};

struct Barriers {
  uint64_t q_full;
  uint64_t slot_full[kMaxSlots];
  uint64_t slot_empty[kMaxSlots];
  uint64_t s_full[2];  // per S buffer
  uint64_t p_full[2];  // per S buffer
  uint64_t pv_done;
  uint64_t o_final;
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

// Visible key interval [lo, hi] of query row q (empty when lo > hi).
struct RowRange {
  int lo, hi;
};

__device__ __forceinline__ RowRange row_range(const FwdParams& p, int q) {
  const long long pos = static_cast<long long>(q) + p.Nk - p.Nq;
  long long lo = 0, hi = static_cast<long long>(p.Nk) - 1;
  if (p.window_left >= 0) lo = max(lo, pos - p.window_left);
  if (p.causal) hi = min(hi, pos);
  if (p.window_right >= 0) hi = min(hi, pos + p.window_right);
  RowRange r;
  r.lo = static_cast<int>(min(lo, static_cast<long long>(p.Nk)));
  r.hi = static_cast<int>(max(hi, -1ll));
  return r;
}

// Waits without checking the abort flag (used only to drain work in flight).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  int dummy = 0;
  mbar_wait(bar, parity, &dummy);
}

template <typename T, int D>
__device__ void producer(const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV, uint8_t* sQ,
                         uint8_t* sKV, Barriers* bars, int b, int h, int q0, int f, int l) {
  using C = Cfg<D>;
  volatile int* abort = &bars->abort;
  const uint64_t pol_q = l2_policy_evict_first();
  const uint64_t pol_kv = l2_policy_evict_last();
  mbar_arrive_expect_tx(&bars->q_full, C::kTileBytes);
#pragma unroll
  for (int ch = 0; ch < D / 64; ++ch)
    tma_load_4d(tmQ, &bars->q_full, sQ + ch * C::kChunkBytes, ch * 64, h, q0, b, pol_q);
  // load order K(f), V(f), K(f+1), V(f+1), ... (the MMA thread acquires
  // V(j) then K(j+1) in each step, which is the same sequence)
  uint32_t it = 0;
  bool ok = true;
  for (int j = f; j <= l && ok; ++j) {
#pragma unroll
    for (int kv = 0; kv < 2; ++kv) {
      const uint32_t slot = it % C::kSlots, n = it / C::kSlots;
      if (n > 0 && !mbar_wait(&bars->slot_empty[slot], (n - 1) & 1, abort)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(&bars->slot_full[slot], C::kTileBytes);
      const CUtensorMap* map = kv ? tmV : tmK;
#pragma unroll
      for (int ch = 0; ch < D / 64; ++ch)
        tma_load_4d(map, &bars->slot_full[slot], sKV + slot * C::kTileBytes + ch * C::kChunkBytes, ch * 64, h,
                    j * BN, b, pol_kv);
      ++it;
    }
  }
  // Every load issued must land before the CTA may exit. On the normal path
  // they all have (the MMA thread consumed them); after an abort, wait.
  drain_wait(&bars->q_full, 0);
  const uint32_t first = it > static_cast<uint32_t>(C::kSlots) ? it - C::kSlots : 0;
  for (uint32_t i = first; i < it; ++i) drain_wait(&bars->slot_full[i % C::kSlots], (i / C::kSlots) & 1);
}

template <typename T, int D>
__device__ void mma_issuer(uint8_t* sQ, uint8_t* sKV, Barriers* bars, uint32_t tmem, int f, int l, bool negate) {
  using C = Cfg<D>;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  // a negative softmax scale is applied as -Q K^T (A-negate bit) times |scale|
  const uint32_t idesc_qk = instr_desc_f16(kBf16, BM, BN, false) | (negate ? (1u << 13) : 0u);
  constexpr uint32_t idesc_pv = instr_desc_f16(kBf16, BM, D, true);
  volatile int* abort = &bars->abort;
  const uint32_t sQaddr = smem_addr(sQ);
  const uint32_t sKVaddr = smem_addr(sKV);

  uint32_t it = 0;
  auto acquire = [&](uint32_t& addr, uint32_t& slot) -> bool {
    slot = it % C::kSlots;
    const bool ok = mbar_wait(&bars->slot_full[slot], (it / C::kSlots) & 1, abort);
    addr = sKVaddr + slot * C::kTileBytes;
    ++it;
    return ok;
  };
  // S(j) = Q K_j^T into S buffer (j - f) & 1: M = 128 query rows, N = 128
  // keys, K = d in steps of 16. Both operands are K-major, 128-byte
  // swizzled, 64 elements per 16 KB chunk.
  auto qk = [&](int j, uint32_t kaddr) {
    const uint32_t d_t = tmem + ((j - f) & 1) * 128;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t off = (kk / 4) * C::kChunkBytes + (kk % 4) * 32;
      mma_ss(d_t, smem_desc_sw128(sQaddr + off, 16, 1024), smem_desc_sw128(kaddr + off, 16, 1024), idesc_qk,
             kk > 0 ? 1u : 0u);
    }
    tc_commit(&bars->s_full[(j - f) & 1]);
  };
  // O (+)= P(j) V_j: A = P from TMEM (16-bit, two keys per column), B = V
  // tile stored keys x d with d contiguous (MN-major): 16 keys = 2048 bytes,
  // the second 64-wide d chunk lies 16 KB further (leading byte offset).
  auto pv = [&](int j, uint32_t vaddr) {
    const uint32_t a_t = tmem + ((j - f) & 1) * 128;
#pragma unroll
    for (int kk = 0; kk < BN / 16; ++kk)
      mma_ts(tmem + kTmemO, a_t + kk * 8, smem_desc_sw128(vaddr + kk * 2048, C::kChunkBytes, 1024), idesc_pv,
             (j > f || kk > 0) ? 1u : 0u);
    tc_commit(&bars->pv_done);
    if (j == l) tc_commit(&bars->o_final);
  };

  bool ok = mbar_wait(&bars->q_full, 0, abort);
  uint32_t aK = 0, slotK = 0, aV = 0, slotV = 0;
  if (ok && (ok = acquire(aK, slotK))) {
    qk(f, aK);
    tc_commit(&bars->slot_empty[slotK]);
  }
  for (int j = f; j <= l && ok; ++j) {
    const bool next = j < l;
    if (!(ok = acquire(aV, slotV))) break;
    if (next) {
      // the next tile's scores go into the other S buffer; its previous
      // contents (P(j-1)) were consumed by the PV product issued last step
      if (!(ok = acquire(aK, slotK))) break;
      qk(j + 1, aK);
      tc_commit(&bars->slot_empty[slotK]);
    }
    if (!(ok = mbar_wait(&bars->p_full[(j - f) & 1], ((j - f) >> 1) & 1, abort))) break;
    tc_fence_after();
    pv(j, aV);
    tc_commit(&bars->slot_empty[slotV]);
  }
  // All MMAs of this thread must be complete before TMEM is released.
  tc_commit(&bars->mma_done);
  drain_wait(&bars->mma_done, 0);
}

// Score transform of one element in log2 units (softcap and ALiBi paths).
template <bool kCap, bool kAlibi>
__device__ __forceinline__ float mod_score(const FwdParams& p, float x, float slope_l2, int dist) {
  float t = kCap ? p.cap_log2 * tanh_via_exp2(x * p.cap_scale) : x * p.scale_log2;
  if (kAlibi) t -= slope_l2 * fabsf(static_cast<float>(dist));
  return t;
}

// The softmax warpgroup: one query row per thread, row == TMEM lane.
// kCap / kAlibi select the score modifiers at compile time; whether a K tile
// needs the element mask is decided per tile for the whole group, so the
// common interior tiles run without per-element compares.
template <typename T, int D, bool kCap, bool kAlibi>
__device__ void softmax_group(const FwdParams& p, Barriers* bars, uint32_t tmem, int b, int h, int q0, bool has,
                              int f, int l) {
  constexpr bool kPlain = !kCap && !kAlibi;
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int r = warp * 32 + lane;  // row of the tile == TMEM lane
  const int q = q0 + r;
  const bool row_ok = q < p.Nq;
  const RowRange rr = row_range(p, row_ok ? q : p.Nq - 1);
  // tile-level bounds: a K tile needs no mask when every row of the tile
  // sees all of it (rows' intervals are monotone in q)
  const int qz = min(q0 + BM - 1, p.Nq - 1);
  const RowRange first_row = row_range(p, q0), last_row = row_range(p, qz);
  const int pos = q + p.Nk - p.Nq;
  const uint32_t lane_sel = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tO = tmem + lane_sel + kTmemO;
  const float slope_l2 = kAlibi ? p.slopes[h] * kLog2e : 0.0f;
  const float sl2 = p.scale_log2;  // >= 0 (a negative scale is folded into the MMA)

  float m = -INFINITY;  // running max (log2 units)
  float lsum = 0.0f;    // running sum of exp2(t - m)
  bool ok = true;
  const int n = has ? l - f + 1 : 0;
  for (int it = 0; it < n; ++it) {
    const int j = f + it;
    const uint32_t tS = tmem + lane_sel + (it & 1) * 128;
    ok = mbar_wait(&bars->s_full[it & 1], (it >> 1) & 1, abort);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    tc_fence_after();
    uint32_t s[4][32];
    const int key0 = j * BN;
    const bool masked = key0 < last_row.lo || key0 + BN - 1 > first_row.hi;  // uniform over the tile
    // pass 1: transform (modifier paths) and tile max. S arrives in two
    // halves so the second TMEM load overlaps the first half's work; four
    // independent 3-input max chains keep the pipes busy.
    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    auto half_max = [&](int c0) {
#pragma unroll
      for (int c = c0; c < c0 + 2; ++c) {
        if (!kPlain || masked) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            float x = __uint_as_float(s[c][e]);
            const int key = key0 + 32 * c + e;
            if (!kPlain) x = mod_score<kCap, kAlibi>(p, x, slope_l2, pos - key);
            if (masked) x = (key >= rr.lo && key <= rr.hi) ? x : -INFINITY;
            s[c][e] = __float_as_uint(x);
          }
        }
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          const int a = (e / 8) & 3;
          mx[a] = fmax3(mx[a], __uint_as_float(s[c][e]), __uint_as_float(s[c][e + 1]));
          mx[a] = fmax3(mx[a], __uint_as_float(s[c][e + 2]), __uint_as_float(s[c][e + 3]));
          mx[a] = fmax3(mx[a], __uint_as_float(s[c][e + 4]), __uint_as_float(s[c][e + 5]));
          mx[a] = fmax3(mx[a], __uint_as_float(s[c][e + 6]), __uint_as_float(s[c][e + 7]));
        }
      }
    };
    tmem_ld32(tS, s[0]);
    tmem_ld32(tS + 32, s[1]);
    tmem_wait_ld();
    reg_fence(s[0]);
    reg_fence(s[1]);
    tmem_ld32(tS + 64, s[2]);
    tmem_ld32(tS + 96, s[3]);
    half_max(0);
    tmem_wait_ld();
    reg_fence(s[2]);
    reg_fence(s[3]);
    half_max(2);
    float mt = fmaxf(fmax3(mx[0], mx[1], mx[2]), mx[3]);
    // plain path: the max was taken over raw scores; scale after (sl2 >= 0)
    if (kPlain) mt = (mt == -INFINITY) ? -INFINITY : mt * sl2;

    // lazy max update
    const float m_new = fmaxf(m, mt);
    float alpha = 1.0f;
    bool rescale = false;
    if (m == -INFINITY) {
      m = m_new;  // nothing accumulated yet for this row (O row is 0, l is 0)
    } else if (m_new > m + kRescaleThreshold) {
      alpha = ex2(m - m_new);
      m = m_new;
      rescale = true;
    }
    lsum *= alpha;
    const float m_eff = (m == -INFINITY) ? 0.0f : m;
    // pass 2: P = exp2(t - m) into the first 64 columns of this S buffer.
    // Pairs of elements go through packed fp32x2 instructions: one FMA
    // (scale and subtract the max) and one add (row sum) per pair.
    const uint64_t m2 = f2_pack(-m_eff, -m_eff);
    const uint64_t mul2 = kPlain ? f2_pack(sl2, sl2) : f2_pack(1.0f, 1.0f);
    uint64_t rsum2[4] = {0, 0, 0, 0};  // independent packed partial sums (0 bits = +0.0f)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float x0 = __uint_as_float(s[c][2 * e]);
        const float x1 = __uint_as_float(s[c][2 * e + 1]);
        float a0, a1;
        f2_unpack(f2_fma(f2_pack(x0, x1), mul2, m2), a0, a1);
        float p0 = ex2(a0), p1 = ex2(a1);
        if (kPlain && masked) {
          // masked entries hold -inf; -inf * 0 would be NaN, so select them out
          p0 = (x0 == -INFINITY) ? 0.0f : p0;
          p1 = (x1 == -INFINITY) ? 0.0f : p1;
        }
        rsum2[e & 3] = f2_add(rsum2[e & 3], f2_pack(p0, p1));
        pk[e] = pack2<T>(p0, p1);
      }
      tmem_st16(tS + 16 * c, pk);
    }
    float r0, r1, r2, r3;
    f2_unpack(f2_add(rsum2[0], rsum2[1]), r0, r1);
    f2_unpack(f2_add(rsum2[2], rsum2[3]), r2, r3);
    const float rs = (r0 + r1) + (r2 + r3);
    if (__any_sync(0xffffffffu, rescale)) {
      // O must be idle: wait for the product of the previous tile (the only
      // one that can still be running).
      if (it > 0) {
        ok = mbar_wait(&bars->pv_done, (it - 1) & 1, abort);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
      }
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * cc, o);
        tmem_wait_ld();
        reg_fence(o);
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
        tmem_st32(tO + 32 * cc, o);
      }
    }
    lsum += rs;
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->p_full[it & 1]);
  }
  if (ok && n > 0) {
    ok = mbar_wait(&bars->o_final, 0, abort);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
  }

  // epilogue: O / l -> dtype, LSE = (m + log2 l) ln 2
  T* orow = reinterpret_cast<T*>(p.out) + ((static_cast<size_t>(b) * p.Nq + (row_ok ? q : 0)) * p.H + h) * D;
  const float inv = lsum > 0.0f ? 1.0f / lsum : 0.0f;
  const float nan = __int_as_float(0x7fc00000);
  if (ok && n > 0) {
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t o[32];
      tmem_ld32(tO + 32 * cc, o);
      tmem_wait_ld();
      reg_fence(o);
      if (row_ok) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack2<T>(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
        uint4* dst = reinterpret_cast<uint4*>(orow + 32 * cc);
#pragma unroll
        for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
      }
    }
  } else if (row_ok) {
    const float fill = ok ? 0.0f : nan;
    const uint32_t w = pack2<T>(fill, fill);
    uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
    for (int v = 0; v < D / 8; ++v) dst[v] = make_uint4(w, w, w, w);
  }
  if (row_ok) {
    float lse_v;
    if (!ok) lse_v = nan;
    else if (lsum > 0.0f) lse_v = (m + lg2(lsum)) * kLn2;
    else lse_v = -INFINITY;
    p.lse[(static_cast<size_t>(b) * p.H + h) * p.Nq + q] = lse_v;
  }
}

template <typename T, int D, bool kCap, bool kAlibi>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::kTileBytes;
  Barriers* bars = reinterpret_cast<Barriers*>(sKV + C::kSlots * C::kTileBytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // 1-D grid, the Q tiles of one (b, h) adjacent so they share K/V in L2;
  // within a head the longest causal work is dispatched first.
  const int bh = static_cast<int>(blockIdx.x) / p.num_tiles;
  const int tile = p.num_tiles - 1 - static_cast<int>(blockIdx.x) % p.num_tiles;
  const int b = bh / p.H, h = bh % p.H;
  const int q0 = tile * BM;

  // K/V tile range of the Q tile (rows' visible intervals are monotone in q)
  const int qz = min(q0 + BM - 1, p.Nq - 1);
  const RowRange ra = row_range(p, q0), rz = row_range(p, qz);
  const bool has = ra.lo <= rz.hi;
  const int f = has ? ra.lo / BN : 0;
  const int l = has ? rz.hi / BN : -1;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < C::kSlots; ++i) {
      mbar_init(&bars->slot_full[i], 1);
      mbar_init(&bars->slot_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 4);
    }
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->o_final, 1);
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < 4) {
    softmax_group<T, D, kCap, kAlibi>(p, bars, tmem, b, h, q0, has, f, l);
  } else if (warp == kProducerWarp) {
    if (lane == 0 && has) producer<T, D>(&tmQ, &tmK, &tmV, sQ, sKV, bars, b, h, q0, f, l);
  } else {
    if (lane == 0 && has) mma_issuer<T, D>(sQ, sKV, bars, tmem, f, l, p.negate_scores != 0);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <typename T, int D, bool kCap, bool kAlibi>
cudaError_t launch(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV, const FwdParams& p,
                   cudaStream_t stream) {
  using C = Cfg<D>;
  static_assert(sizeof(Barriers) <= 1024, "barrier block exceeds its reserve");
  static_assert(C::kSmemBytes <= 232448, "shared memory budget exceeded");
  static_assert(C::kSlots <= kMaxSlots, "too many K/V slots");
  auto kernel = fwd_kernel<T, D, kCap, kAlibi>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.num_tiles * p.B * p.H);
  kernel<<<grid, kThreads, C::kSmemBytes, stream>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_mods(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV, const FwdParams& p,
                        cudaStream_t stream) {
  const bool alibi = p.slopes != nullptr;
  if (p.use_softcap) return alibi ? launch<T, D, true, true>(tmQ, tmK, tmV, p, stream)
                                  : launch<T, D, true, false>(tmQ, tmK, tmV, p, stream);
  return alibi ? launch<T, D, false, true>(tmQ, tmK, tmV, p, stream)
               : launch<T, D, false, false>(tmQ, tmK, tmV, p, stream);
}

}  // namespace

cudaError_t launch_fwd(bool bf16, int d, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                       const FwdParams& p, cudaStream_t stream) {
  if (bf16) return d == 128 ? launch_mods<__nv_bfloat16, 128>(tmQ, tmK, tmV, p, stream)
                            : launch_mods<__nv_bfloat16, 64>(tmQ, tmK, tmV, p, stream);
  return d == 128 ? launch_mods<__half, 128>(tmQ, tmK, tmV, p, stream)
                  : launch_mods<__half, 64>(tmQ, tmK, tmV, p, stream);
}

}  // namespace fa

