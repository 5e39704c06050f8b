// fa_decode_kernel.cu -- split-KV ("flash-decoding") attention of one query
// token over a paged KV cache, plus the merge of the split partials.
//
// Method ("Flash-Attention v2.0 到 v2.7 更新", section v2.2: instead of one
// block walking the whole KV, the KV cache is cut along the sequence, each
// block takes one piece and an extra kernel merges the pieces; section v2.5:
// the cache is non-contiguous and addressed through a block table;
// "FlashAttention深度解析", section on inference: with a short query the goal
// is to load the KV cache as efficiently as possible).
//
// The split kernel is bound by HBM bandwidth (about 1 flop per byte), so it
// is written for the memory system rather than the tensor cores: every lane
// issues 16-byte loads, the d/8 lanes that share one token read its 2*d-byte
// row in one coalesced transaction, and each lane keeps U tokens' K and V
// loads in flight before it touches any of them. One CTA (4 warps) handles
// one (sequence, head, split); its tokens are interleaved across warps in
// groups of U*32/(d/8) tokens. Per token: page = block_table[b][t / page],
// row = t % page; the dot product is reduced across the token's lanes with
// shuffles; the online softmax keeps (m, l, acc) per lane group and the four
// warps' states are merged through shared memory at the end. Page sizes that
// are a multiple of 64 take a TMA-staged variant of the split kernel (below);
// other page sizes use the direct 16-byte-load variant.
#include "fa_internal.h"
#include "sm100_ptx.cuh"

#include <type_traits>

namespace fa {
namespace {

constexpr int kWarps = 4;
constexpr int kUnroll = 4;

__device__ __forceinline__ uint4 load_stream(const void* ptr) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(ptr));
  return v;
}

template <typename T>
__device__ __forceinline__ void widen8(const uint4& v, float (&f)[8]) {
  const float2 a = unpack2<T>(v.x), b = unpack2<T>(v.y), c = unpack2<T>(v.z), d = unpack2<T>(v.w);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
  f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

// Key range [t0, t1) of split s: the visible keys [lo, hi) cut into
// num_splits near-equal chunks whose length is a whole number of pages.
__device__ __forceinline__ void split_range(int lo, int hi, int num_splits, int s, int page, int& t0, int& t1) {
  t0 = t1 = hi;
  if (hi <= lo) return;
  const long long n = hi - lo;
  long long chunk = (n + num_splits - 1) / num_splits;
  chunk = (chunk + page - 1) / page * page;
  const long long a = lo + static_cast<long long>(s) * chunk;
  t0 = static_cast<int>(min(a, static_cast<long long>(hi)));
  t1 = static_cast<int>(min(a + chunk, static_cast<long long>(hi)));
}

template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32) decode_split_kernel(const DecodeParams p) {
  constexpr int LPT = D / 8;    // lanes per token
  constexpr int TPW = 32 / LPT; // tokens per warp per load step
  constexpr int kStep = kWarps * TPW * kUnroll;
  __shared__ float sm_m[kWarps], sm_l[kWarps];
  __shared__ float sm_acc[kWarps][D];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane / LPT;   // token slot within the warp
  const int cl = lane % LPT;  // 8-element chunk of the head dimension
  const int h = blockIdx.x % p.H;
  const int s = blockIdx.x / p.H;
  const int b = blockIdx.y;

  const int L_raw = p.cache_seqlens[b];
  const long long max_len = static_cast<long long>(p.max_blocks) * p.page_size;
  bool bad = L_raw < 0 || L_raw > max_len;
  const int L = bad ? 0 : L_raw;
  const int pos = L - 1;  // the query's key position (bottom-right alignment)
  const int lo = p.window_left >= 0 ? max(0, pos - p.window_left) : 0;
  int t0, t1;
  split_range(lo, L, p.num_splits, s, p.page_size, t0, t1);

  // query chunk, pre-scaled so the dot product is already in its final units
  float qf[8];
  widen8<T>(*reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.q) +
                                            (static_cast<size_t>(b) * p.H + h) * D + cl * 8),
            qf);
  const float qscale = p.use_softcap ? p.cap_scale : p.scale_log2;
#pragma unroll
  for (int e = 0; e < 8; ++e) qf[e] *= qscale;
  const bool alibi = p.slopes != nullptr;
  const float slope_l2 = alibi ? p.slopes[h] * kLog2e : 0.0f;

  const size_t tok_stride = static_cast<size_t>(p.H_kv) * D;  // elements
  const size_t page_stride = static_cast<size_t>(p.page_size) * tok_stride;
  const int hk = h / (p.H / p.H_kv);  // cache head of query head h
  const T* kbase = reinterpret_cast<const T*>(p.k_cache) + static_cast<size_t>(hk) * D + cl * 8;
  const T* vbase = reinterpret_cast<const T*>(p.v_cache) + static_cast<size_t>(hk) * D + cl * 8;
  const int* bt = p.block_table + static_cast<size_t>(b) * p.max_blocks;

  float m = -INFINITY, lsum = 0.0f;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0f;

  for (int base = t0 + warp * TPW * kUnroll; base < t1; base += kStep) {
    uint4 kr[kUnroll], vr[kUnroll];
    bool valid[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int tok = base + u * TPW + g;
      valid[u] = tok < t1;
      kr[u] = vr[u] = make_uint4(0, 0, 0, 0);
      if (valid[u]) {
        const int pg = bt[tok / p.page_size];
        if (pg < 0 || pg >= p.num_pages) {
          bad = true;
          valid[u] = false;
        } else {
          const size_t off = static_cast<size_t>(pg) * page_stride + static_cast<size_t>(tok % p.page_size) * tok_stride;
          kr[u] = load_stream(kbase + off);
          vr[u] = load_stream(vbase + off);
        }
      }
    }
    float sc[kUnroll];
    float mt = -INFINITY;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float kf[8];
      widen8<T>(kr[u], kf);
      float dot = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) dot = fmaf(qf[e], kf[e], dot);
#pragma unroll
      for (int o = LPT / 2; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      float t = p.use_softcap ? p.cap_log2 * tanh_via_exp2(dot) : dot;
      const int tok = base + u * TPW + g;
      if (alibi) t -= slope_l2 * static_cast<float>(pos - tok);
      sc[u] = valid[u] ? t : -INFINITY;
      mt = fmaxf(mt, sc[u]);
    }
    const float m_new = fmaxf(m, mt);
    if (m_new == -INFINITY) continue;  // nothing visible yet in this lane group
    const float alpha = ex2(m - m_new);
    lsum *= alpha;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] *= alpha;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const float pu = ex2(sc[u] - m_new);
      lsum += pu;
      float vf[8];
      widen8<T>(vr[u], vf);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = fmaf(pu, vf[e], acc[e]);
    }
    m = m_new;
  }

  // merge the TPW lane groups of this warp
#pragma unroll
  for (int o = LPT; o < 32; o <<= 1) {
    const float m_o = __shfl_xor_sync(0xffffffffu, m, o);
    const float l_o = __shfl_xor_sync(0xffffffffu, lsum, o);
    const float mm = fmaxf(m, m_o);
    const float a = (m == -INFINITY) ? 0.0f : ex2(m - mm);
    const float a_o = (m_o == -INFINITY) ? 0.0f : ex2(m_o - mm);
    lsum = lsum * a + l_o * a_o;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float x_o = __shfl_xor_sync(0xffffffffu, acc[e], o);
      acc[e] = acc[e] * a + x_o * a_o;
    }
    m = mm;
  }
  if (lane < LPT) {
#pragma unroll
    for (int e = 0; e < 8; ++e) sm_acc[warp][cl * 8 + e] = acc[e];
  }
  if (lane == 0) {
    sm_m[warp] = m;
    sm_l[warp] = lsum;
  }
  const bool any_bad = __syncthreads_or(bad) != 0;

  // merge the warps; thread c owns output element c
  const int c = threadIdx.x;
  if (c >= D) return;
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm_m[w]);
  float ltot = 0.0f, oc = 0.0f;
  if (M != -INFINITY) {
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float a = (sm_m[w] == -INFINITY) ? 0.0f : ex2(sm_m[w] - M);
      ltot += sm_l[w] * a;
      oc += sm_acc[w][c] * a;
    }
  }
  const float nan = __int_as_float(0x7fc00000);
  float o_val, lse_val;
  if (any_bad) {
    o_val = nan;
    lse_val = nan;
  } else if (ltot > 0.0f) {
    o_val = oc / ltot;
    lse_val = (M + lg2(ltot)) * kLn2;
  } else {
    o_val = 0.0f;
    lse_val = -INFINITY;
  }
  const size_t row = static_cast<size_t>(b) * p.H + h;
  if (p.num_splits == 1) {
    T* out = reinterpret_cast<T*>(p.out) + row * D;
    if constexpr (std::is_same<T, __nv_bfloat16>::value) out[c] = __float2bfloat16_rn(o_val);
    else out[c] = __float2half_rn(o_val);
    if (c == 0) p.lse[row] = lse_val;
  } else {
    const size_t prow = static_cast<size_t>(s) * p.B * p.H + row;
    p.o_part[prow * D + c] = o_val;
    if (c == 0) p.lse_part[prow] = lse_val;
  }
}

// Merge of the split partials of one (sequence, head): lse = ln sum_s exp(lse_s),
// O = sum_s exp(lse_s - lse) O_s; empty splits (lse_s = -inf) weigh nothing,
// a NaN partial (invalid block-table entry) makes the row NaN.
template <typename T, int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const DecodeParams p) {
  const int row = blockIdx.x;  // b * H + h
  const int c = threadIdx.x;
  const int BH = p.B * p.H;
  const int S = p.num_splits;
  float M = -INFINITY;
  bool nan_in = false;
  for (int s = 0; s < S; ++s) {
    const float x = p.lse_part[static_cast<size_t>(s) * BH + row];
    nan_in |= (x != x);
    M = fmaxf(M, x);
  }
  const float nan = __int_as_float(0x7fc00000);
  float o_val = 0.0f, lse_val = -INFINITY;
  if (nan_in) {
    o_val = lse_val = nan;
  } else if (M != -INFINITY) {
    float wsum = 0.0f, oc = 0.0f;
    for (int s = 0; s < S; ++s) {
      const size_t prow = static_cast<size_t>(s) * BH + row;
      const float w = ex2((p.lse_part[prow] - M) * kLog2e);
      wsum += w;
      oc += w * p.o_part[prow * D + c];
    }
    o_val = oc / wsum;
    lse_val = M + lg2(wsum) * kLn2;
  }
  T* out = reinterpret_cast<T*>(p.out) + static_cast<size_t>(row) * D;
  if constexpr (std::is_same<T, __nv_bfloat16>::value) out[c] = __float2bfloat16_rn(o_val);
  else out[c] = __float2half_rn(o_val);
  if (c == 0) p.lse[row] = lse_val;
}

// Split kernel for page sizes that are a multiple of 64: a producer lane
// streams each 64-token slice of a page (K and V, one TMA box each, no
// multicast) into a ring of shared-memory stages; four consumer warps read
// the rows with 16-byte shared loads. Every global byte of K and V moves in
// whole 2*d-byte rows and the producer keeps up to kStages*32 KB in flight
// per CTA, two CTAs per SM.
constexpr int kRows = 64;  // tokens per stage

template <int D, int G = 1>
struct TmaCfg {
  // grouped-query CTAs (G > 1) keep fewer stages so three fit on an SM
  static constexpr int kStages = (D == 128) ? (G > 1 ? 2 : 3) : (G > 1 ? 4 : 6);
  static constexpr int kTile = kRows * D * 2;  // bytes of one K (or V) stage
  static constexpr int kShared = 4096 + 3 * kWarps * 4 * D * 4 / 4;  // barrier block, up to 4 heads
  static constexpr int kSmem = 2 * kStages * kTile + kShared;
};

template <int D, int G>
struct TmaShared {
  uint64_t full[TmaCfg<D, G>::kStages];
  uint64_t empty[TmaCfg<D, G>::kStages];
  int bad[TmaCfg<D, G>::kStages];
  int abort;
  float m[kWarps][G], l[kWarps][G];
  float acc[kWarps][G][D];
};

// G query heads per CTA (grouped-query attention: heads that share one cache
// head read its K/V stream once). CTA slot hs of a (sequence, split) serves
// query heads hs*G .. hs*G + G - 1, which all map to cache head
// hs*G / (H / H_kv). G = 1 is the plain per-head kernel.
template <typename T, int D, int G>
__global__ void __launch_bounds__((kWarps + 1) * 32, G > 1 ? 3 : 2)
    decode_split_tma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                            const DecodeParams p) {
  using C = TmaCfg<D, G>;
  constexpr int NST = C::kStages;
  constexpr int LPT = D / 8;                  // lanes per token
  constexpr int TPW = 32 / LPT;               // tokens per warp per step
  constexpr int kSteps = kRows / kWarps / TPW; // steps per stage per warp (16 tokens a warp)
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sK = smem;
  uint8_t* sV = smem + NST * C::kTile;
  TmaShared<D, G>* sh = reinterpret_cast<TmaShared<D, G>*>(smem + 2 * NST * C::kTile);
  volatile int* abort = &sh->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slots = p.H / G;
  const int h0 = (blockIdx.x % slots) * G;  // first query head of this CTA
  const int hk = h0 / (p.H / p.H_kv);        // their cache head
  const int s = blockIdx.x / slots;
  const int b = blockIdx.y;
  const int L_raw = p.cache_seqlens[b];
  const long long max_len = static_cast<long long>(p.max_blocks) * p.page_size;
  bool bad = L_raw < 0 || L_raw > max_len;
  const int L = bad ? 0 : L_raw;
  const int pos = L - 1;
  const int lo = p.window_left >= 0 ? max(0, pos - p.window_left) : 0;
  int t0, t1;
  split_range(lo, L, p.num_splits, s, p.page_size, t0, t1);
  const int a0 = (t0 / kRows) * kRows;
  const int n_st = t1 > t0 ? (t1 - a0 + kRows - 1) / kRows : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&sh->full[i], 1);
      mbar_init(&sh->empty[i], kWarps);
      sh->bad[i] = 0;
    }
    sh->abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kWarps) {
    // ---------------- producer
    if (lane == 0 && n_st > 0) {
      const uint64_t pol = l2_policy_evict_first();
      const int* bt = p.block_table + static_cast<size_t>(b) * p.max_blocks;
      int issued = 0;
      for (int i = 0; i < n_st; ++i) {
        const int slot = i % NST, n = i / NST;
        if (n > 0 && !mbar_wait(&sh->empty[slot], (n - 1) & 1, abort)) break;
        const int a = a0 + i * kRows;
        const int pg = bt[a / p.page_size];
        if (pg < 0 || pg >= p.num_pages) {
          sh->bad[slot] = 1;  // never dereferenced; consumers turn it into NaN rows
          mbar_arrive(&sh->full[slot]);
        } else {
          sh->bad[slot] = 0;
          mbar_arrive_expect_tx(&sh->full[slot], 2 * C::kTile);
          tma_load_4d(&tmK, &sh->full[slot], sK + slot * C::kTile, 0, hk, a % p.page_size, pg, pol);
          tma_load_4d(&tmV, &sh->full[slot], sV + slot * C::kTile, 0, hk, a % p.page_size, pg, pol);
        }
        issued = i + 1;
      }
      // loads in flight must land before the CTA exits
      const int first = issued > NST ? issued - NST : 0;
      int dummy = 0;
      for (int i = first; i < issued; ++i) mbar_wait(&sh->full[i % NST], (i / NST) & 1, &dummy);
    }
  } else if constexpr (G > 1) {
    // ---------------- consumers, G heads: the per-head partial dot products
    // of a token are reduce-scattered over its LPT lanes, so each lane ends
    // with the full score of one head (lanes of a token group split into G
    // subgroups of LPT / G lanes, subgroup j holding head j); the lane keeps
    // that head's running max and sum, and broadcasts its probabilities to
    // the other lanes of the token group for the V update.
    const int g = lane / LPT;
    const int cl = lane % LPT;
    const int gbase = lane & ~(LPT - 1);  // first lane of this token group
    constexpr int SUB = LPT / G;           // lanes per head subgroup
    const int my = cl / SUB;               // the head this lane scores
    const float qscale = p.use_softcap ? p.cap_scale : p.scale_log2;
    const bool alibi = p.slopes != nullptr;
    // q and the accumulators as packed fp32 pairs (fp32x2 FMA)
    uint64_t q2[G][4];
    uint64_t acc2[G][4];
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
      float qf[8];
      widen8<T>(*reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.q) +
                                                (static_cast<size_t>(b) * p.H + h0 + gi) * D + cl * 8),
                qf);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        q2[gi][e] = f2_pack(qf[2 * e] * qscale, qf[2 * e + 1] * qscale);
        acc2[gi][e] = 0;  // 0 bits = +0.0f pair
      }
    }
    const float slope_l2 = alibi ? p.slopes[h0 + my] * kLog2e : 0.0f;
    float m = -INFINITY, lsum = 0.0f;  // of head `my`, this token group

    for (int i = 0; i < n_st; ++i) {
      const int slot = i % NST;
      bool ok = mbar_wait(&sh->full[slot], (i / NST) & 1, abort);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        bad = true;
        break;
      }
      if (sh->bad[slot]) {
        bad = true;
      } else {
        const T* kt = reinterpret_cast<const T*>(sK + slot * C::kTile);
        const T* vt = reinterpret_cast<const T*>(sV + slot * C::kTile);
        const int a = a0 + i * kRows;
        float sc[kSteps];
        float mt = -INFINITY;
#pragma unroll
        for (int st = 0; st < kSteps; ++st) {
          const int r = warp * (kRows / kWarps) + st * TPW + g;
          float kf[8];
          widen8<T>(*reinterpret_cast<const uint4*>(kt + r * D + cl * 8), kf);
          uint64_t k2[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) k2[e] = f2_pack(kf[2 * e], kf[2 * e + 1]);
          float v[G];
#pragma unroll
          for (int gi = 0; gi < G; ++gi) {
            uint64_t d2 = f2_mul(q2[gi][0], k2[0]);
#pragma unroll
            for (int e = 1; e < 4; ++e) d2 = f2_fma(q2[gi][e], k2[e], d2);
            float d0, d1;
            f2_unpack(d2, d0, d1);
            v[gi] = d0 + d1;
          }
          // reduce-scatter over the token's lanes
          float s1;
          if constexpr (G == 4) {
            const bool up = (cl & (LPT / 2)) != 0;
            const float a0s = up ? v[0] : v[2], a1s = up ? v[1] : v[3];
            const float k0 = up ? v[2] : v[0], k1 = up ? v[3] : v[1];
            const float r0 = k0 + __shfl_xor_sync(0xffffffffu, a0s, LPT / 2);
            const float r1 = k1 + __shfl_xor_sync(0xffffffffu, a1s, LPT / 2);
            const bool up2 = (cl & (LPT / 4)) != 0;
            s1 = (up2 ? r1 : r0) + __shfl_xor_sync(0xffffffffu, up2 ? r0 : r1, LPT / 4);
          } else {
            const bool up = (cl & (LPT / 2)) != 0;
            s1 = (up ? v[1] : v[0]) + __shfl_xor_sync(0xffffffffu, up ? v[0] : v[1], LPT / 2);
          }
#pragma unroll
          for (int o = SUB / 2; o >= 1; o >>= 1) s1 += __shfl_xor_sync(0xffffffffu, s1, o);
          const int tok = a + r;
          float t = p.use_softcap ? p.cap_log2 * tanh_via_exp2(s1) : s1;
          if (alibi) t -= slope_l2 * static_cast<float>(pos - tok);
          sc[st] = (tok >= t0 && tok < t1) ? t : -INFINITY;
          mt = fmaxf(mt, sc[st]);
        }
        const float mn = fmaxf(m, mt);
        float pw[kSteps];
        float alpha = 1.0f;
        if (mn != -INFINITY) {
          alpha = ex2(m - mn);
          lsum *= alpha;
#pragma unroll
          for (int st = 0; st < kSteps; ++st) {
            pw[st] = ex2(sc[st] - mn);
            lsum += pw[st];
          }
          m = mn;
        } else {
#pragma unroll
          for (int st = 0; st < kSteps; ++st) pw[st] = 0.0f;
        }
        // every lane updates all G heads for its 8 columns of V
#pragma unroll
        for (int gi = 0; gi < G; ++gi) {
          const float al = __shfl_sync(0xffffffffu, alpha, gbase + gi * SUB);
          const uint64_t al2 = f2_pack(al, al);
#pragma unroll
          for (int e = 0; e < 4; ++e) acc2[gi][e] = f2_mul(acc2[gi][e], al2);
        }
#pragma unroll
        for (int st = 0; st < kSteps; ++st) {
          const int r = warp * (kRows / kWarps) + st * TPW + g;
          float vf[8];
          widen8<T>(*reinterpret_cast<const uint4*>(vt + r * D + cl * 8), vf);
          uint64_t v2[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) v2[e] = f2_pack(vf[2 * e], vf[2 * e + 1]);
#pragma unroll
          for (int gi = 0; gi < G; ++gi) {
            const float pg = __shfl_sync(0xffffffffu, pw[st], gbase + gi * SUB);
            const uint64_t pg2 = f2_pack(pg, pg);
#pragma unroll
            for (int e = 0; e < 4; ++e) acc2[gi][e] = f2_fma(v2[e], pg2, acc2[gi][e]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->empty[slot]);
    }
    // merge the token groups of this warp per head, then publish
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
      float acc[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) f2_unpack(acc2[gi][e], acc[2 * e], acc[2 * e + 1]);
      float mg = __shfl_sync(0xffffffffu, m, gbase + gi * SUB);
      float lg = __shfl_sync(0xffffffffu, lsum, gbase + gi * SUB);
#pragma unroll
      for (int o = LPT; o < 32; o <<= 1) {
        const float m_o = __shfl_xor_sync(0xffffffffu, mg, o);
        const float l_o = __shfl_xor_sync(0xffffffffu, lg, o);
        const float mm = fmaxf(mg, m_o);
        const float x = (mg == -INFINITY) ? 0.0f : ex2(mg - mm);
        const float x_o = (m_o == -INFINITY) ? 0.0f : ex2(m_o - mm);
        lg = lg * x + l_o * x_o;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float a_o = __shfl_xor_sync(0xffffffffu, acc[e], o);
          acc[e] = acc[e] * x + a_o * x_o;
        }
        mg = mm;
      }
      if (lane < LPT) {
#pragma unroll
        for (int e = 0; e < 8; ++e) sh->acc[warp][gi][cl * 8 + e] = acc[e];
      }
      if (lane == 0) {
        sh->m[warp][gi] = mg;
        sh->l[warp][gi] = lg;
      }
    }
  } else {
    // ---------------- consumers, one head: the kSteps partial dot products a
    // lane holds for its token group are reduce-scattered over the group's
    // LPT lanes, so lane cl ends with the full score of step cl / R (R = LPT /
    // kSteps lanes share a step); scores, the running max and the sum are
    // then worked once per token instead of on every lane, and the step's
    // probability is broadcast back to the group for the V update.
    static_assert(G == 1, "grouped-query CTAs take the branch above");
    static_assert(LPT % kSteps == 0, "a token group needs a lane per step");
    constexpr int R = LPT / kSteps;
    const int g = lane / LPT;
    const int cl = lane % LPT;
    const int gbase = lane & ~(LPT - 1);
    const int my_st = cl / R;  // the step whose score this lane ends up with
    const float qscale = p.use_softcap ? p.cap_scale : p.scale_log2;
    const bool alibi = p.slopes != nullptr;
    uint64_t q2[4], acc2[4];
    {
      float qf[8];
      widen8<T>(*reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.q) +
                                                (static_cast<size_t>(b) * p.H + h0) * D + cl * 8),
                qf);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        q2[e] = f2_pack(qf[2 * e] * qscale, qf[2 * e + 1] * qscale);
        acc2[e] = 0;  // +0.0f pair
      }
    }
    const float slope_l2 = alibi ? p.slopes[h0] * kLog2e : 0.0f;
    float m = -INFINITY, lsum = 0.0f;  // lsum: this lane's steps only

    for (int i = 0; i < n_st; ++i) {
      const int slot = i % NST;
      bool ok = mbar_wait(&sh->full[slot], (i / NST) & 1, abort);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        bad = true;
        break;
      }
      if (sh->bad[slot]) {
        bad = true;
      } else {
        const T* kt = reinterpret_cast<const T*>(sK + slot * C::kTile);
        const T* vt = reinterpret_cast<const T*>(sV + slot * C::kTile);
        const int a = a0 + i * kRows;
        float dv[kSteps];
#pragma unroll
        for (int st = 0; st < kSteps; ++st) {
          const int r = warp * (kRows / kWarps) + st * TPW + g;
          float kf[8];
          widen8<T>(*reinterpret_cast<const uint4*>(kt + r * D + cl * 8), kf);
          uint64_t d2 = f2_mul(q2[0], f2_pack(kf[0], kf[1]));
#pragma unroll
          for (int e = 1; e < 4; ++e) d2 = f2_fma(q2[e], f2_pack(kf[2 * e], kf[2 * e + 1]), d2);
          float d0, d1;
          f2_unpack(d2, d0, d1);
          dv[st] = d0 + d1;
        }
        // reduce-scatter: at each level the lane keeps the half of its steps
        // named by its lane bit and adds the partner's copy of that half
#pragma unroll
        for (int n = kSteps, off = LPT / 2; n > 1; n >>= 1, off >>= 1) {
          const bool up = (cl & off) != 0;
#pragma unroll
          for (int j = 0; j < n / 2; ++j) {
            const float keep = up ? dv[j + n / 2] : dv[j];
            const float send = up ? dv[j] : dv[j + n / 2];
            dv[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
          }
        }
#pragma unroll
        for (int off = R / 2; off >= 1; off >>= 1) dv[0] += __shfl_xor_sync(0xffffffffu, dv[0], off);
        const int tok = a + warp * (kRows / kWarps) + my_st * TPW + g;
        float t = p.use_softcap ? p.cap_log2 * tanh_via_exp2(dv[0]) : dv[0];
        if (alibi) t -= slope_l2 * static_cast<float>(pos - tok);
        const float sc = (tok >= t0 && tok < t1) ? t : -INFINITY;
        float mt = sc;
#pragma unroll
        for (int off = R; off < LPT; off <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
        const float mn = fmaxf(m, mt);
        const bool live = mn != -INFINITY;  // uniform over the token group
        const float alpha = live ? ex2(m - mn) : 1.0f;
        const float pw = live ? ex2(sc - mn) : 0.0f;
        lsum = lsum * alpha + pw;
        m = live ? mn : m;
        const uint64_t al2 = f2_pack(alpha, alpha);
#pragma unroll
        for (int e = 0; e < 4; ++e) acc2[e] = f2_mul(acc2[e], al2);
#pragma unroll
        for (int st = 0; st < kSteps; ++st) {
          const int r = warp * (kRows / kWarps) + st * TPW + g;
          float vf[8];
          widen8<T>(*reinterpret_cast<const uint4*>(vt + r * D + cl * 8), vf);
          const float ps = __shfl_sync(0xffffffffu, pw, gbase + st * R);
          const uint64_t p2 = f2_pack(ps, ps);
#pragma unroll
          for (int e = 0; e < 4; ++e) acc2[e] = f2_fma(f2_pack(vf[2 * e], vf[2 * e + 1]), p2, acc2[e]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->empty[slot]);
    }
    // the group's sum over its distinct steps, then merge the token groups of
    // this warp and publish the warp's state
#pragma unroll
    for (int off = R; off < LPT; off <<= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
    float acc[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) f2_unpack(acc2[e], acc[2 * e], acc[2 * e + 1]);
#pragma unroll
    for (int o = LPT; o < 32; o <<= 1) {
      const float m_o = __shfl_xor_sync(0xffffffffu, m, o);
      const float l_o = __shfl_xor_sync(0xffffffffu, lsum, o);
      const float mm = fmaxf(m, m_o);
      const float x = (m == -INFINITY) ? 0.0f : ex2(m - mm);
      const float x_o = (m_o == -INFINITY) ? 0.0f : ex2(m_o - mm);
      lsum = lsum * x + l_o * x_o;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float a_o = __shfl_xor_sync(0xffffffffu, acc[e], o);
        acc[e] = acc[e] * x + a_o * x_o;
      }
      m = mm;
    }
    if (lane < LPT) {
#pragma unroll
      for (int e = 0; e < 8; ++e) sh->acc[warp][0][cl * 8 + e] = acc[e];
    }
    if (lane == 0) {
      sh->m[warp][0] = m;
      sh->l[warp][0] = lsum;
    }
  }
  const bool any_bad = __syncthreads_or(bad) != 0;

  const int c = threadIdx.x;
  if (c >= D) return;
  const float nan = __int_as_float(0x7fc00000);
#pragma unroll
  for (int gi = 0; gi < G; ++gi) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sh->m[w][gi]);
    float ltot = 0.0f, oc = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float x = (sh->m[w][gi] == -INFINITY) ? 0.0f : ex2(sh->m[w][gi] - M);
        ltot += sh->l[w][gi] * x;
        oc += sh->acc[w][gi][c] * x;
      }
    }
    float o_val, lse_val;
    if (any_bad) {
      o_val = nan;
      lse_val = nan;
    } else if (ltot > 0.0f) {
      o_val = oc / ltot;
      lse_val = (M + lg2(ltot)) * kLn2;
    } else {
      o_val = 0.0f;
      lse_val = -INFINITY;
    }
    const size_t row = static_cast<size_t>(b) * p.H + h0 + gi;
    if (p.num_splits == 1) {
      T* out = reinterpret_cast<T*>(p.out) + row * D;
      if constexpr (std::is_same<T, __nv_bfloat16>::value) out[c] = __float2bfloat16_rn(o_val);
      else out[c] = __float2half_rn(o_val);
      if (c == 0) p.lse[row] = lse_val;
    } else {
      const size_t prow = static_cast<size_t>(s) * p.B * p.H + row;
      p.o_part[prow * D + c] = o_val;
      if (c == 0) p.lse_part[prow] = lse_val;
    }
  }
}

template <typename T, int D>
cudaError_t launch(const DecodeParams& p, const CUtensorMap* tmK, const CUtensorMap* tmV, cudaStream_t stream) {
  dim3 grid(p.H * p.num_splits, p.B);
  if (tmK != nullptr) {
    // query heads per CTA: the largest of 4, 2, 1 that divides the group
    const int group = p.H / p.H_kv;
    const int G = group % 4 == 0 ? 4 : (group % 2 == 0 ? 2 : 1);
    auto go = [&](auto g_tag) -> cudaError_t {
      constexpr int kG = decltype(g_tag)::value;
      using C = TmaCfg<D, kG>;
      static_assert(sizeof(TmaShared<D, kG>) <= C::kShared, "decode shared block exceeds its reserve");
      auto kernel = decode_split_tma_kernel<T, D, kG>;
      cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
      if (e != cudaSuccess) return e;
      dim3 g2(p.H / kG * p.num_splits, p.B);
      kernel<<<g2, (kWarps + 1) * 32, C::kSmem, stream>>>(*tmK, *tmV, p);
      return cudaSuccess;
    };
    cudaError_t e = G == 4 ? go(std::integral_constant<int, 4>{})
                           : (G == 2 ? go(std::integral_constant<int, 2>{}) : go(std::integral_constant<int, 1>{}));
    if (e != cudaSuccess) return e;
  } else {
    decode_split_kernel<T, D><<<grid, kWarps * 32, 0, stream>>>(p);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || p.num_splits == 1) return e;
  decode_combine_kernel<T, D><<<p.B * p.H, D, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(bool bf16, int d, const DecodeParams& p, const CUtensorMap* tmK, const CUtensorMap* tmV,
                          cudaStream_t stream) {
  if (bf16) return d == 128 ? launch<__nv_bfloat16, 128>(p, tmK, tmV, stream)
                            : launch<__nv_bfloat16, 64>(p, tmK, tmV, stream);
  return d == 128 ? launch<__half, 128>(p, tmK, tmV, stream) : launch<__half, 64>(p, tmK, tmV, stream);
}

}  // namespace fa
