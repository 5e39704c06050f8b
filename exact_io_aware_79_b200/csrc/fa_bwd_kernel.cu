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
// Kernels: bwd_rowdot (D, one warp per 32 / (d/8) rows), bwd_kernel (one CTA
// per 64-key block of one (b, cache head): dK and dV stay in registers while
// the CTA walks the query blocks of every query head that reads the cache
// head; dQ partials are added into an fp32 accumulator by TMA reduce-add),
// bwd_dq_cast (dQ =
// scale * accumulator, to the input type). The deterministic mode (the
// pages' version 2.4 names a deterministic backward) drops the atomic dQ
// partials and runs bwd_dq_kernel instead, which sums dQ over the key blocks
// of each query block in a fixed order; every output then repeats bit for bit.
//
// bwd_kernel's products are warp-level m16n8k16 tensor-core MMAs; each of the
// four warps owns 16 keys (the rows of its products). K, V and the double-
// buffered Q and dO tiles arrive by TMA as 64-column boxes with 128-byte
// swizzle, so each 16-byte chunk c of row r sits at chunk c ^ (r % 8) of its
// 128-byte line. Fragment bookkeeping (g = lane / 4, t = lane % 4, perm(n) =
// n / 2 + 4 (n % 2)):
//  * S^T = K Q^T and dP^T = V dO^T: product row g (g + 8) is key 16 w +
//    perm(g) (+ 8); column n of query n-tile j is query 8 j + perm(n). The
//    head-dimension order is permuted so each lane's operands are whole
//    16-byte chunks (chunk 4 i + t of a row feeds k-steps 2 i and 2 i + 1,
//    words 0-1 and 2-3), which the sum over k does not notice; perm keeps the
//    two rows a quarter-warp reads in opposite halves of a swizzle line.
//  * dV += P^T dO and dK += dS^T Q: the accumulators of query n-tiles 2 k and
//    2 k + 1 are the A operand of k-step k (queries 16 k + perm(0..7), then
//    16 k + 8 + perm(0..7)); ldmatrix.trans reads the matching dO / Q rows.
//  * dQ = dS K: dS^T is stored to shared memory (row = key, column = query in
//    the n-tile order above); ldmatrix.trans turns it into the A operand with
//    queries as rows, K (rows = keys in natural order) is the B operand.
#include "fa_bwd_common.cuh"
#include "fa_internal.h"
#include "sm100_ptx.cuh"

#include <type_traits>

namespace fa {
namespace {

constexpr int kBwdWarps = 4;
constexpr int kBlk = 64;  // keys per CTA, queries per step
// each CTA thread fetches one of the block's 64 lse and 64 D values
static_assert(kBwdWarps * 32 == 2 * kBlk, "row-vector fetch assumes two values per query row per thread pair");

__device__ __forceinline__ int perm8(int n) { return (n >> 1) | ((n & 1) << 2); }

// Byte offset of 16-byte chunk c of row r in a 64-row tile of 64-column
// boxes with 128-byte swizzle.
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
  return static_cast<uint32_t>((c >> 3) * (kBlk * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

template <int D>
struct BwdCfg {
  static constexpr int kTile = kBlk * D * 2;  // one 64-row tile of K, V, Q or dO
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTile;
  static constexpr int kOffQ = 2 * kTile;   // two buffers
  static constexpr int kOffO = 4 * kTile;   // two buffers (dO)
  static constexpr int kOffS = 6 * kTile;   // dS^T, 64 x 64 16-bit
  static constexpr int kOffL = kOffS + kBlk * kBlk * 2;  // [2 buffers][lse * log2(e) x 64, D x 64] fp32
  static constexpr int kOffBar = kOffL + 4 * kBlk * 4;
  static constexpr int kSmem = 1024 + kOffBar + 64;  // + slack to align to 1 KB
};

// D_i = sum_c dO_ic O_ic in fp32, [B, H, Nq]; outside the deterministic mode
// the same threads zero the fp32 dQ accumulator's rows (their 8 columns).
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

// Is key j visible to the query at key position pos (the forward's rule)?
__device__ __forceinline__ bool key_visible(int pos, int j, int Nk, const BwdParams& p) {
  if (j >= Nk) return false;
  if (p.causal && j > pos) return false;
  if (p.window_left >= 0 && j < pos - p.window_left) return false;
  if (p.window_right >= 0 && j > pos + p.window_right) return false;
  return true;
}

// Outside the deterministic mode the CTA also adds its dQ partials into the
// fp32 accumulator; in it bwd_dq_kernel forms dQ instead.
template <typename T, int D>
__global__ void __launch_bounds__(kBwdWarps * 32, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
               const __grid_constant__ CUtensorMap tmDQ, const BwdParams p) {
  using C = BwdCfg<D>;
  constexpr int KS = D / 16;  // k-steps over the head dimension
  constexpr int NT = D / 8;   // n-tiles over the head dimension
  constexpr int NH = NT / 2;  // n-tiles per half of the dQ product
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint8_t* sS = smem + C::kOffS;
  float* sL = reinterpret_cast<float*>(smem + C::kOffL);        // [2][lse * log2(e) x 64, D x 64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);  // full[2], kv
  int* abort_flag = reinterpret_cast<int*>(bars + 3);
  volatile int* abort = abort_flag;
  const uint32_t sK_a = smem_addr(sK), sS_a = smem_addr(sS);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int kb = blockIdx.x;
  const int b = blockIdx.y / p.H_kv, hk = blockIdx.y % p.H_kv;
  const int G = p.H / p.H_kv;
  const int k0 = kb * kBlk;
  int Nq, Nk;
  long long qrow, krow;
  if (!bwd_seq(p, b, Nq, Nk, qrow, krow) || k0 >= Nk) return;  // uniform over the CTA
  // tensor-map coordinates: (row, batch) = (q, b) for fixed lengths, (qrow + q, 0) packed
  const int tb = p.cu_q == nullptr ? b : 0;
  const int tq0 = p.cu_q == nullptr ? 0 : static_cast<int>(qrow);
  const int tk0 = p.cu_q == nullptr ? 0 : static_cast<int>(krow);
  const int off = Nk - Nq;  // query i sits at key position i + off

  // query rows that can see a key of [k0, k1)
  const int k1 = min(k0 + kBlk, Nk);
  long long q_lo = 0, q_hi = Nq - 1;
  {
    int right = -1;  // keys j <= pos + right are the only visible ones (when >= 0)
    if (p.causal) right = 0;
    if (p.window_right >= 0) right = p.causal ? min(0, p.window_right) : p.window_right;
    if (p.causal || p.window_right >= 0) q_lo = max(q_lo, static_cast<long long>(k0) - off - right);
    if (p.window_left >= 0) q_hi = min(q_hi, static_cast<long long>(k1 - 1) + p.window_left - off);
  }
  const int qb_lo = q_lo <= q_hi ? static_cast<int>(q_lo / kBlk) : 0;
  const int n_qb = q_lo <= q_hi ? static_cast<int>(q_hi / kBlk) - qb_lo + 1 : 0;
  const int n_it = G * n_qb;

  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_init(&bars[2], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const uint64_t pol = l2_policy_evict_last();
  auto issue = [&](int it) {
    const int buf = it & 1;
    const int h = hk * G + it / n_qb;
    const int q0 = (qb_lo + it % n_qb) * kBlk;
    mbar_arrive_expect_tx(&bars[buf], 2 * C::kTile);
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh) {
      tma_load_4d(&tmQ, &bars[buf], smem + C::kOffQ + buf * C::kTile + hh * kBlk * 128, hh * 64, h, tq0 + q0, tb,
                  pol);
      tma_load_4d(&tmO, &bars[buf], smem + C::kOffO + buf * C::kTile + hh * kBlk * 128, hh * 64, h, tq0 + q0, tb,
                  pol);
    }
  };
  if (threadIdx.x == 0 && n_it > 0) {
    mbar_arrive_expect_tx(&bars[2], 2 * C::kTile);
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh) {
      tma_load_4d(&tmK, &bars[2], sK + hh * kBlk * 128, hh * 64, hk, tk0 + k0, tb, pol);
      tma_load_4d(&tmV, &bars[2], sV + hh * kBlk * 128, hh * 64, hk, tk0 + k0, tb, pol);
    }
    issue(0);
    if (n_it > 1) issue(1);
  }

  float dv[NT][4], dk[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dv[n][e] = dk[n][e] = 0.0f;

  const int krow0 = warp * 16 + perm8(gq);  // this lane's product rows: krow0, krow0 + 8
  const bool alibi = p.slopes != nullptr;
  const bool dq_on = !p.deterministic;
  bool failed = false;
  int issued = n_it > 1 ? 2 : n_it;
  bool reload_pending = false;  // thread 0: a dQ reduce still reads this block's Q/dO buffers

  // the row vectors (lse, D) of iteration `it`: thread x < 64 fetches lse of
  // query q0 + x, thread 64 + x its D; read one iteration ahead into a register
  auto fetch_rowvec = [&](int it) -> float {
    const int h = hk * G + it / n_qb;
    const int q = (qb_lo + it % n_qb) * kBlk + (threadIdx.x & (kBlk - 1));
    if (q >= Nq) return threadIdx.x < kBlk ? -INFINITY : 0.0f;
    const size_t ri = rowvec_index(p, b, h, qrow, q);
    return threadIdx.x < kBlk ? p.lse[ri] * kLog2e : p.dvec[ri];
  };
  float rv_next = n_it > 0 ? fetch_rowvec(0) : 0.0f;

#pragma unroll 1
  for (int it = 0; it < n_it; ++it) {
    const int buf = it & 1;
    const int h = hk * G + it / n_qb;
    const int q0 = (qb_lo + it % n_qb) * kBlk;
    const float slope2 = alibi ? p.slopes[h] * kLog2e : 0.0f;
    sL[buf * 2 * kBlk + threadIdx.x] = rv_next;  // [buf][lse 0..63 | D 0..63]
    if (it + 1 < n_it) rv_next = fetch_rowvec(it + 1);
    bool ok = true;
    if (it == 0) ok = mbar_wait(&bars[2], 0, abort);
    ok = ok && mbar_wait(&bars[buf], (it >> 1) & 1, abort);
    // one barrier: row vectors visible, tiles landed everywhere, and every
    // warp done with the previous block's dS tile
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    if (threadIdx.x == 0 && reload_pending) {
      // the previous block's dQ boxes have been read out of its Q/dO buffers
      // by now (a block of compute ago at most): reload them
      bulk_wait_read_all();
      if (issued < n_it) {
        issue(issued);
        ++issued;
      }
      reload_pending = false;
    }
    const uint8_t* sQ = smem + C::kOffQ + buf * C::kTile;
    const uint8_t* sO = smem + C::kOffO + buf * C::kTile;
    const uint32_t sQ_a = smem_addr(sQ), sO_a = smem_addr(sO);
    const float* lse2 = sL + buf * 2 * kBlk;
    const float* dvec = lse2 + kBlk;
    // every (key, query) pair of this block pair visible?
    bool full = k0 + kBlk <= Nk && q0 + kBlk <= Nq;
    if (p.causal || p.window_right >= 0) {
      const int right = p.window_right >= 0 ? (p.causal ? min(0, p.window_right) : p.window_right) : 0;
      full = full && k0 + kBlk - 1 <= q0 + off + right;
    }
    if (p.window_left >= 0) full = full && k0 >= q0 + kBlk - 1 + off - p.window_left;

#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      // ---- S^T and dP^T for query n-tiles 4 hf .. 4 hf + 3
      float sc[4][4], dp[4][4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[jj][e] = dp[jj][e] = 0.0f;
#pragma unroll
      for (int i = 0; i < KS / 2; ++i) {
        const int c = 4 * i + tq;
        const uint4 k0v = *reinterpret_cast<const uint4*>(sK + sw_off(krow0, c));
        const uint4 k1v = *reinterpret_cast<const uint4*>(sK + sw_off(krow0 + 8, c));
        const uint4 v0v = *reinterpret_cast<const uint4*>(sV + sw_off(krow0, c));
        const uint4 v1v = *reinterpret_cast<const uint4*>(sV + sw_off(krow0 + 8, c));
        const uint32_t ka0[4] = {k0v.x, k1v.x, k0v.y, k1v.y}, ka1[4] = {k0v.z, k1v.z, k0v.w, k1v.w};
        const uint32_t va0[4] = {v0v.x, v1v.x, v0v.y, v1v.y}, va1[4] = {v0v.z, v1v.z, v0v.w, v1v.w};
        uint4 qw[4], ow[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int r = 8 * (4 * hf + jj) + perm8(gq);
          qw[jj] = *reinterpret_cast<const uint4*>(sQ + sw_off(r, c));
          ow[jj] = *reinterpret_cast<const uint4*>(sO + sw_off(r, c));
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          mma_16816<T>(sc[jj], ka0, qw[jj].x, qw[jj].y);
          mma_16816<T>(dp[jj], va0, ow[jj].x, ow[jj].y);
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          mma_16816<T>(sc[jj], ka1, qw[jj].z, qw[jj].w);
          mma_16816<T>(dp[jj], va1, ow[jj].z, ow[jj].w);
        }
      }
      // ---- P and dS, elementwise (sc <- P, dp <- dS); blocks with every
      // (key, query) pair visible skip the per-element mask
      auto elementwise = [&](auto masked_tag) {
        constexpr bool kMasked = decltype(masked_tag)::value;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int key = k0 + krow0 + 8 * (e >> 1);
            const int ql = 8 * (4 * hf + jj) + tq + 4 * (e & 1);
            const int pos = q0 + ql + off;
            float logit2, dfac = 1.0f;
            if (p.use_softcap) {
              const float th = tanh_via_exp2(sc[jj][e] * p.cap_scale);
              logit2 = th * p.cap_log2;
              dfac = 1.0f - th * th;
            } else {
              logit2 = sc[jj][e] * p.scale_log2;
            }
            if (alibi) logit2 -= slope2 * fabsf(static_cast<float>(pos - key));
            float pr = ex2(logit2 - lse2[ql]);
            if constexpr (kMasked) {
              if (!(q0 + ql < Nq && key_visible(pos, key, Nk, p))) pr = 0.0f;
            }
            sc[jj][e] = pr;
            dp[jj][e] = pr * (dp[jj][e] - dvec[ql]) * dfac;
          }
        }
      };
      if (full) elementwise(std::false_type{});
      else elementwise(std::true_type{});
      // ---- dV += P^T dO, dK += dS^T Q over the query k-steps 2 hf, 2 hf + 1
#pragma unroll
      for (int kx = 0; kx < 2; ++kx) {
        const int kk = 2 * hf + kx;
        const uint32_t pa[4] = {pack2<T>(sc[2 * kx][0], sc[2 * kx][1]), pack2<T>(sc[2 * kx][2], sc[2 * kx][3]),
                                pack2<T>(sc[2 * kx + 1][0], sc[2 * kx + 1][1]),
                                pack2<T>(sc[2 * kx + 1][2], sc[2 * kx + 1][3])};
        const uint32_t da[4] = {pack2<T>(dp[2 * kx][0], dp[2 * kx][1]), pack2<T>(dp[2 * kx][2], dp[2 * kx][3]),
                                pack2<T>(dp[2 * kx + 1][0], dp[2 * kx + 1][1]),
                                pack2<T>(dp[2 * kx + 1][2], dp[2 * kx + 1][3])};
        const int brow = 16 * kk + ((lane >> 3) & 1) * 8 + perm8(lane & 7);
#pragma unroll
        for (int u = 0; u < NT / 2; ++u) {
          const int cc = 2 * u + (lane >> 4);
          uint32_t bo[4], bq[4];
          ldsm_x4_trans(bo, sO_a + sw_off(brow, cc));
          ldsm_x4_trans(bq, sQ_a + sw_off(brow, cc));
          mma_16816<T>(dv[2 * u], pa, bo[0], bo[1]);
          mma_16816<T>(dv[2 * u + 1], pa, bo[2], bo[3]);
          mma_16816<T>(dk[2 * u], da, bq[0], bq[1]);
          mma_16816<T>(dk[2 * u + 1], da, bq[2], bq[3]);
        }
      }
      // ---- dS^T to shared memory: row = key (local), column = query position
#pragma unroll
      for (int jj = 0; jj < 4 && dq_on; ++jj) {
        const int jt = 4 * hf + jj;
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int kr = krow0 + 8 * hr;
          *reinterpret_cast<uint32_t*>(sS + kr * 128 + ((jt ^ (kr & 7)) << 4) + 4 * tq) =
              pack2<T>(dp[jj][2 * hr], dp[jj][2 * hr + 1]);
        }
      }
    }
    __syncthreads();  // dS^T complete; this block's Q and dO buffers are free
    if (dq_on) {
      // ---- dQ (rows = query positions 16 w .. 16 w + 15) = dS K, in two halves of n-tiles,
      // staged as fp32 in this block's idle Q and dO buffers (64-row boxes of 32 columns,
      // 128-byte swizzle) and added into the accumulator by TMA reduce-add
      uint8_t* stage[2] = {smem + C::kOffQ + buf * C::kTile, smem + C::kOffO + buf * C::kTile};
      constexpr int kBoxesPerBuf = D / 64;  // 8 KB fp32 boxes per 16-bit tile buffer
#pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
        float acc[NH][4];
#pragma unroll
        for (int n = 0; n < NH; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk) {
          const int mi = lane >> 3;
          const int akey = 16 * kk + (mi >> 1) * 8 + (lane & 7);
          const int achunk = 2 * warp + (mi & 1);
          uint32_t a[4];
          ldsm_x4_trans(a, sS_a + akey * 128 + ((achunk ^ (akey & 7)) << 4));
          const int brow = 16 * kk + (mi & 1) * 8 + (lane & 7);
#pragma unroll
          for (int u = 0; u < NH / 2; ++u) {
            const int cc = nh * NH + 2 * u + (lane >> 4);
            uint32_t bk[4];
            ldsm_x4_trans(bk, sK_a + sw_off(brow, cc));
            mma_16816<T>(acc[2 * u], a, bk[0], bk[1]);
            mma_16816<T>(acc[2 * u + 1], a, bk[2], bk[3]);
          }
        }
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int row = 16 * warp + 8 * hr + perm8(gq);
#pragma unroll
          for (int n = 0; n < NH; ++n) {
            const int col = nh * NH * 8 + 8 * n + 2 * tq;
            const int box = col >> 5, bcol = col & 31;
            uint8_t* dst = stage[box / kBoxesPerBuf] + (box % kBoxesPerBuf) * (kBlk * 128) + row * 128 +
                           ((((bcol >> 2) ^ (row & 7))) << 4) + (bcol & 3) * 4;
            *reinterpret_cast<float2*>(dst) = make_float2(acc[n][2 * hr], acc[n][2 * hr + 1]);
          }
        }
      }
      fence_proxy_async_shared();
      __syncthreads();
      if (threadIdx.x == 0) {
#pragma unroll
        for (int box = 0; box < D / 32; ++box)
          tma_reduce_add_4d(&tmDQ, stage[box / kBoxesPerBuf] + (box % kBoxesPerBuf) * (kBlk * 128), box * 32, h,
                            tq0 + q0, tb);
        bulk_commit_group();
        reload_pending = true;  // the staging buffers are reloaded after the next barrier
      }
    } else if (threadIdx.x == 0 && issued < n_it) {
      issue(issued);
      ++issued;
    }
  }
  if (threadIdx.x == 0) bulk_wait_all();
  // loads still in flight must land before the CTA exits
  if (threadIdx.x == 0 && failed) {
    int dummy = 0;
    for (int i = max(0, issued - 2); i < issued; ++i) mbar_wait(&bars[i & 1], (i >> 1) & 1, &dummy);
    mbar_wait(&bars[2], 0, &dummy);
  }

  // ---- dK (scaled) and dV rows of this lane: keys k0 + krow0 (+ 8)
  const float nan = __int_as_float(0x7fc00000);
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int key = k0 + krow0 + 8 * hr;
    if (key >= Nk) continue;
    const size_t base = static_cast<size_t>(krow + key) * p.dkv_tok + static_cast<size_t>(hk) * D + 2 * tq;
    T* dk_out = reinterpret_cast<T*>(p.dk) + base;
    T* dv_out = reinterpret_cast<T*>(p.dv) + base;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const float k0f = failed ? nan : dk[n][2 * hr] * p.scale, k1f = failed ? nan : dk[n][2 * hr + 1] * p.scale;
      const float v0f = failed ? nan : dv[n][2 * hr], v1f = failed ? nan : dv[n][2 * hr + 1];
      *reinterpret_cast<uint32_t*>(dk_out + 8 * n) = pack2<T>(k0f, k1f);
      *reinterpret_cast<uint32_t*>(dv_out + 8 * n) = pack2<T>(v0f, v1f);
    }
  }
}

// Deterministic dQ: one CTA per 64-query block of one (b, query head); each
// warp owns 16 queries and walks the visible key blocks in increasing order,
// rebuilding S = Q K^T and dP = dO V^T, so dQ = scale * sum_j dS K is summed
// in a fixed order (no atomics). Fragment bookkeeping mirrors bwd_kernel with
// the roles of keys and queries swapped: product row g (g + 8) is query
// 16 w + perm(g) (+ 8), column n of key n-tile j is key 8 j + perm(n).
template <int D>
struct DqCfg {
  static constexpr int kTile = kBlk * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffO = kTile;
  static constexpr int kOffK = 2 * kTile;  // two buffers
  static constexpr int kOffV = 4 * kTile;  // two buffers
  static constexpr int kOffBar = 6 * kTile;
  static constexpr int kSmem = 1024 + kOffBar + 64;
};

template <typename T, int D>
__global__ void __launch_bounds__(kBwdWarps * 32, 2)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const BwdParams p) {
  using C = DqCfg<D>;
  constexpr int KS = D / 16;
  constexpr int NT = D / 8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint8_t* sQ = smem + C::kOffQ;
  const uint8_t* sO = smem + C::kOffO;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);  // full[2], q
  int* abort_flag = reinterpret_cast<int*>(bars + 3);
  volatile int* abort = abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int qb = blockIdx.x;
  const int b = blockIdx.y / p.H, h = blockIdx.y % p.H;
  const int hk = h / (p.H / p.H_kv);
  const int q0 = qb * kBlk;
  int Nq, Nk;
  long long qrow, krow;
  if (!bwd_seq(p, b, Nq, Nk, qrow, krow) || q0 >= Nq) return;  // uniform over the CTA
  const int tb = p.cu_q == nullptr ? b : 0;
  const int tq0 = p.cu_q == nullptr ? 0 : static_cast<int>(qrow);
  const int tk0 = p.cu_q == nullptr ? 0 : static_cast<int>(krow);
  const int off = Nk - Nq;

  // key blocks that hold a key visible to a query of [q0, qmax]
  const int qmax = min(q0 + kBlk - 1, Nq - 1);
  long long k_lo = 0, k_hi = Nk - 1;
  if (p.causal || p.window_right >= 0) {
    const int right = p.window_right >= 0 ? (p.causal ? min(0, p.window_right) : p.window_right) : 0;
    k_hi = min(k_hi, static_cast<long long>(qmax) + off + right);
  }
  if (p.window_left >= 0) k_lo = max(k_lo, static_cast<long long>(q0) + off - p.window_left);
  const int kb_lo = k_lo <= k_hi ? static_cast<int>(k_lo / kBlk) : 0;
  const int n_it = k_lo <= k_hi ? static_cast<int>(k_hi / kBlk) - kb_lo + 1 : 0;

  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_init(&bars[2], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const uint64_t pol = l2_policy_evict_last();
  auto issue = [&](int it) {
    const int buf = it & 1;
    const int k0 = (kb_lo + it) * kBlk;
    mbar_arrive_expect_tx(&bars[buf], 2 * C::kTile);
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh) {
      tma_load_4d(&tmK, &bars[buf], smem + C::kOffK + buf * C::kTile + hh * kBlk * 128, hh * 64, hk, tk0 + k0, tb,
                  pol);
      tma_load_4d(&tmV, &bars[buf], smem + C::kOffV + buf * C::kTile + hh * kBlk * 128, hh * 64, hk, tk0 + k0, tb,
                  pol);
    }
  };
  if (threadIdx.x == 0 && n_it > 0) {
    mbar_arrive_expect_tx(&bars[2], 2 * C::kTile);
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh) {
      tma_load_4d(&tmQ, &bars[2], smem + C::kOffQ + hh * kBlk * 128, hh * 64, h, tq0 + q0, tb, pol);
      tma_load_4d(&tmO, &bars[2], smem + C::kOffO + hh * kBlk * 128, hh * 64, h, tq0 + q0, tb, pol);
    }
    issue(0);
    if (n_it > 1) issue(1);
  }

  const int qrow0 = warp * 16 + perm8(gq);  // this lane's product rows: qrow0, qrow0 + 8
  float lse2[2], dvr[2];
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int q = q0 + qrow0 + 8 * hr;
    const size_t ri = rowvec_index(p, b, h, qrow, q);
    lse2[hr] = q < Nq ? p.lse[ri] * kLog2e : -INFINITY;
    dvr[hr] = q < Nq ? p.dvec[ri] : 0.0f;
  }
  const bool alibi = p.slopes != nullptr;
  const float slope2 = alibi ? p.slopes[h] * kLog2e : 0.0f;
  float dq[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) dq[n][0] = dq[n][1] = dq[n][2] = dq[n][3] = 0.0f;
  bool failed = false;
  int issued = n_it > 1 ? 2 : n_it;

#pragma unroll 1
  for (int it = 0; it < n_it; ++it) {
    const int buf = it & 1;
    const int k0 = (kb_lo + it) * kBlk;
    bool ok = true;
    if (it == 0) ok = mbar_wait(&bars[2], 0, abort);
    ok = ok && mbar_wait(&bars[buf], (it >> 1) & 1, abort);
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    const uint8_t* sK = smem + C::kOffK + buf * C::kTile;
    const uint8_t* sV = smem + C::kOffV + buf * C::kTile;
    const uint32_t sK_a = smem_addr(sK);
    bool full = k0 + kBlk <= Nk && q0 + kBlk <= Nq;
    if (p.causal || p.window_right >= 0) {
      const int right = p.window_right >= 0 ? (p.causal ? min(0, p.window_right) : p.window_right) : 0;
      full = full && k0 + kBlk - 1 <= q0 + off + right;
    }
    if (p.window_left >= 0) full = full && k0 >= q0 + kBlk - 1 + off - p.window_left;

#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      // ---- S and dP for key n-tiles 4 hf .. 4 hf + 3
      float sc[4][4], dp[4][4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[jj][e] = dp[jj][e] = 0.0f;
#pragma unroll
      for (int i = 0; i < KS / 2; ++i) {
        const int c = 4 * i + tq;
        const uint4 q0v = *reinterpret_cast<const uint4*>(sQ + sw_off(qrow0, c));
        const uint4 q1v = *reinterpret_cast<const uint4*>(sQ + sw_off(qrow0 + 8, c));
        const uint4 o0v = *reinterpret_cast<const uint4*>(sO + sw_off(qrow0, c));
        const uint4 o1v = *reinterpret_cast<const uint4*>(sO + sw_off(qrow0 + 8, c));
        const uint32_t qa0[4] = {q0v.x, q1v.x, q0v.y, q1v.y}, qa1[4] = {q0v.z, q1v.z, q0v.w, q1v.w};
        const uint32_t oa0[4] = {o0v.x, o1v.x, o0v.y, o1v.y}, oa1[4] = {o0v.z, o1v.z, o0v.w, o1v.w};
        uint4 kw[4], vw[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int r = 8 * (4 * hf + jj) + perm8(gq);
          kw[jj] = *reinterpret_cast<const uint4*>(sK + sw_off(r, c));
          vw[jj] = *reinterpret_cast<const uint4*>(sV + sw_off(r, c));
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          mma_16816<T>(sc[jj], qa0, kw[jj].x, kw[jj].y);
          mma_16816<T>(dp[jj], oa0, vw[jj].x, vw[jj].y);
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          mma_16816<T>(sc[jj], qa1, kw[jj].z, kw[jj].w);
          mma_16816<T>(dp[jj], oa1, vw[jj].z, vw[jj].w);
        }
      }
      // ---- dS, elementwise (dp <- dS)
      auto elementwise = [&](auto masked_tag) {
        constexpr bool kMasked = decltype(masked_tag)::value;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int hr = e >> 1;
            const int ql = qrow0 + 8 * hr;
            const int key = k0 + 8 * (4 * hf + jj) + tq + 4 * (e & 1);
            const int pos = q0 + ql + off;
            float logit2, dfac = 1.0f;
            if (p.use_softcap) {
              const float th = tanh_via_exp2(sc[jj][e] * p.cap_scale);
              logit2 = th * p.cap_log2;
              dfac = 1.0f - th * th;
            } else {
              logit2 = sc[jj][e] * p.scale_log2;
            }
            if (alibi) logit2 -= slope2 * fabsf(static_cast<float>(pos - key));
            float pr = ex2(logit2 - lse2[hr]);
            if constexpr (kMasked) {
              if (!(q0 + ql < Nq && key_visible(pos, key, Nk, p))) pr = 0.0f;
            }
            dp[jj][e] = pr * (dp[jj][e] - dvr[hr]) * dfac;
          }
        }
      };
      if (full) elementwise(std::false_type{});
      else elementwise(std::true_type{});
      // ---- dQ += dS K over the key k-steps 2 hf, 2 hf + 1
#pragma unroll
      for (int kx = 0; kx < 2; ++kx) {
        const int kk = 2 * hf + kx;
        const uint32_t da[4] = {pack2<T>(dp[2 * kx][0], dp[2 * kx][1]), pack2<T>(dp[2 * kx][2], dp[2 * kx][3]),
                                pack2<T>(dp[2 * kx + 1][0], dp[2 * kx + 1][1]),
                                pack2<T>(dp[2 * kx + 1][2], dp[2 * kx + 1][3])};
        const int brow = 16 * kk + ((lane >> 3) & 1) * 8 + perm8(lane & 7);
#pragma unroll
        for (int u = 0; u < NT / 2; ++u) {
          const int cc = 2 * u + (lane >> 4);
          uint32_t bk[4];
          ldsm_x4_trans(bk, sK_a + sw_off(brow, cc));
          mma_16816<T>(dq[2 * u], da, bk[0], bk[1]);
          mma_16816<T>(dq[2 * u + 1], da, bk[2], bk[3]);
        }
      }
    }
    __syncthreads();  // this block's K and V buffers are free
    if (threadIdx.x == 0 && issued < n_it) {
      issue(issued);
      ++issued;
    }
  }
  if (threadIdx.x == 0 && failed) {
    int dummy = 0;
    for (int i = max(0, issued - 2); i < issued; ++i) mbar_wait(&bars[i & 1], (i >> 1) & 1, &dummy);
    mbar_wait(&bars[2], 0, &dummy);
  }
  const float nan = __int_as_float(0x7fc00000);
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int q = q0 + qrow0 + 8 * hr;
    if (q >= Nq) continue;
    T* out = reinterpret_cast<T*>(p.dq) + static_cast<size_t>(qrow + q) * p.dq_tok + static_cast<size_t>(h) * D +
             2 * tq;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const float x0 = failed ? nan : dq[n][2 * hr] * p.scale, x1 = failed ? nan : dq[n][2 * hr + 1] * p.scale;
      *reinterpret_cast<uint32_t*>(out + 8 * n) = pack2<T>(x0, x1);
    }
  }
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
  if constexpr (D == 128) {
    // the tensor-core kernel (its job counter was zeroed by the row-dot kernel)
    e = launch_bwd_tc(std::is_same<T, __nv_bfloat16>::value, p, tmQ, tmK, tmV, tmO, tmDQ, stream);
  } else {
    using C = BwdCfg<D>;
    auto kernel = bwd_kernel<T, D>;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.Nk + kBlk - 1) / kBlk, p.B * p.H_kv);
    kernel<<<grid, kBwdWarps * 32, C::kSmem, stream>>>(tmQ, tmK, tmV, tmO, tmDQ, p);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  if (p.deterministic) {
    // the fixed-order dQ pass: on the tensor cores for d = 128 (its job
    // counter was zeroed by the row-dot kernel), warp-level otherwise
    if constexpr (D == 128) return launch_bwd_dq_tc(std::is_same<T, __nv_bfloat16>::value, p, tmQ, tmK, tmV, tmO, stream);
    using Cq = DqCfg<D>;
    auto dq_kernel = bwd_dq_kernel<T, D>;
    e = cudaFuncSetAttribute(dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Cq::kSmem);
    if (e != cudaSuccess) return e;
    dim3 g2((p.Nq + kBlk - 1) / kBlk, p.B * p.H);
    dq_kernel<<<g2, kBwdWarps * 32, Cq::kSmem, stream>>>(tmQ, tmK, tmV, tmO, p);
    return cudaGetLastError();
  }
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
