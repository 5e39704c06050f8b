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
// other page sizes use the direct 16-byte-load variant. With grouped-query
// caches (several query heads per cache head) the TMA-staged kernel reads a
// cache head once for up to 16 query heads and computes their scores and
// output update as warp-level tensor-core products, since the group's
// arithmetic per K/V byte would otherwise bound it on the FMA pipe.
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

template <int D>
struct TmaCfg {
  static constexpr int kStages = (D == 128) ? 3 : 6;
  static constexpr int kTile = kRows * D * 2;  // bytes of one K (or V) stage
  static constexpr int kShared = 1024 + kWarps * D * 4;  // barriers, flags, per-warp state
  static constexpr int kSmem = 2 * kStages * kTile + kShared;
};

template <int D>
struct TmaShared {
  uint64_t full[TmaCfg<D>::kStages];
  uint64_t empty[TmaCfg<D>::kStages];
  int bad[TmaCfg<D>::kStages];
  int abort;
  float m[kWarps], l[kWarps];
  float acc[kWarps][D];
};

// One (sequence, head, split) per CTA.
template <typename T, int D>
__global__ void __launch_bounds__((kWarps + 1) * 32, 2)
    decode_split_tma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                            const DecodeParams p) {
  using C = TmaCfg<D>;
  constexpr int NST = C::kStages;
  constexpr int LPT = D / 8;                  // lanes per token
  constexpr int TPW = 32 / LPT;               // tokens per warp per step
  constexpr int kSteps = kRows / kWarps / TPW; // steps per stage per warp (16 tokens a warp)
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sK = smem;
  uint8_t* sV = smem + NST * C::kTile;
  TmaShared<D>* sh = reinterpret_cast<TmaShared<D>*>(smem + 2 * NST * C::kTile);
  volatile int* abort = &sh->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h0 = blockIdx.x % p.H;      // query head of this CTA
  const int hk = h0 / (p.H / p.H_kv);  // its cache head
  const int s = blockIdx.x / p.H;
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
  } else {
    // ---------------- consumers, one head: the kSteps partial dot products a
    // lane holds for its token group are reduce-scattered over the group's
    // LPT lanes, so lane cl ends with the full score of step cl / R (R = LPT /
    // kSteps lanes share a step); scores, the running max and the sum are
    // then worked once per token instead of on every lane, and the step's
    // probability is broadcast back to the group for the V update.
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
      for (int e = 0; e < 8; ++e) sh->acc[warp][cl * 8 + e] = acc[e];
    }
    if (lane == 0) {
      sh->m[warp] = m;
      sh->l[warp] = lsum;
    }
  }
  const bool any_bad = __syncthreads_or(bad) != 0;

  const int c = threadIdx.x;
  if (c >= D) return;
  const float nan = __int_as_float(0x7fc00000);
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sh->m[w]);
  float ltot = 0.0f, oc = 0.0f;
  if (M != -INFINITY) {
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float x = (sh->m[w] == -INFINITY) ? 0.0f : ex2(sh->m[w] - M);
      ltot += sh->l[w] * x;
      oc += sh->acc[w][c] * x;
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
  const size_t row = static_cast<size_t>(b) * p.H + h0;
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

// Split kernel for grouped-query caches (page sizes that are a multiple of
// 64): the G <= 16 query heads that share one cache head are the rows of
// warp-level m16n8k16 tensor-core products, so a stage's scores S = Q K^T and
// its update O += P V cost two products per token instead of G dot products
// per token on the FMA pipe. The producer lane streams each 64-token slice of
// a page (K and V, 64-column boxes with 128-byte swizzle, no multicast) into
// a ring of stages; each of the four consumer warps owns 16 tokens of every
// stage and keeps its own online-softmax state (m, l, O) for the group's rows.
//
// Fragment bookkeeping (g = lane / 4, t = lane % 4):
//  * score product, k = head dimension: lane (g, t) of a k-step pair j reads
//    the 16-byte chunk c = 4j + t of its token's K row and uses words 0-1 as
//    the B operand of k-step 2j and words 2-3 for k-step 2j+1; the Q operand
//    is laid out with the same assignment of head-dimension columns, so the
//    sum over k is the full dot product whatever the column order.
//  * column n of n-tile jt is the stage row 16 w + 8 jt + (n / 2 + 4 (n % 2))
//    (w the warp), so the two tokens a quarter-warp reads sit in opposite
//    halves of the 128-byte swizzle row and the loads are conflict-free; the
//    accumulator pair (2t, 2t+1) of n-tile jt is thus rows 16 w + 8 jt + t
//    and + t + 4.
//  * the output product's k = token: the score accumulators of n-tiles 0 and
//    1 are exactly the A operand (P) of one k-step, and ldmatrix.trans reads
//    V's matching rows as the B operand.
constexpr int kMmaRows = 16;

template <int D>
struct MmaCfg {
  static constexpr int kStages = (D == 128) ? 3 : 6;
  static constexpr int kHalf = kRows * 128;        // one 64-token x 64-column swizzled box
  static constexpr int kHalves = D / 64;
  static constexpr int kTile = kHalves * kHalf;    // K (or V) of one stage
  static constexpr int kShared = 1024;             // barriers, flags, per-warp row state
  static constexpr int kSmem = 1024 + 2 * kStages * kTile + kShared;  // + slack to align the ring to 1 KB
};

template <int D>
struct MmaShared {
  uint64_t full[MmaCfg<D>::kStages];
  uint64_t empty[MmaCfg<D>::kStages];
  int bad[MmaCfg<D>::kStages];
  int abort;
  float m[kWarps][kMmaRows], l[kWarps][kMmaRows];
};

template <typename T, int D>
__global__ void __launch_bounds__((kWarps + 1) * 32, 2)
    decode_split_mma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                            const DecodeParams p, const int G) {
  using C = MmaCfg<D>;
  constexpr int NST = C::kStages;
  constexpr int KS = D / 16;  // k-steps of the score product
  constexpr int NT = D / 8;   // n-tiles of the output product
  static_assert(kRows == kWarps * 16, "each consumer warp owns 16 tokens of a stage");
  static_assert(sizeof(MmaShared<D>) <= C::kShared, "decode shared block exceeds its reserve");
  static_assert(kWarps * kMmaRows * D * 4 <= 2 * NST * C::kTile, "the epilogue reuses the ring");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = smem + NST * C::kTile;
  MmaShared<D>* sh = reinterpret_cast<MmaShared<D>*>(smem + 2 * NST * C::kTile);
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
#pragma unroll
          for (int hh = 0; hh < C::kHalves; ++hh) {
            tma_load_4d(&tmK, &sh->full[slot], sK + slot * C::kTile + hh * C::kHalf, hh * 64, hk,
                        a % p.page_size, pg, pol);
            tma_load_4d(&tmV, &sh->full[slot], sV + slot * C::kTile + hh * C::kHalf, hh * 64, hk,
                        a % p.page_size, pg, pol);
          }
        }
        issued = i + 1;
      }
      // loads in flight must land before the CTA exits
      const int first = issued > NST ? issued - NST : 0;
      int dummy = 0;
      for (int i = first; i < issued; ++i) mbar_wait(&sh->full[i % NST], (i / NST) & 1, &dummy);
    }
  } else {
    // ---------------- consumers
    const int gq = lane >> 2, tq = lane & 3;
    const bool real0 = gq < G, real1 = gq + 8 < G;  // product rows gq and gq + 8
    const bool hi = G > 8;
    uint32_t qa[KS][4];
    {
      const T* q0 = reinterpret_cast<const T*>(p.q) + (static_cast<size_t>(b) * p.H + h0 + gq) * D;
      const T* q1 = q0 + 8 * D;
#pragma unroll
      for (int j = 0; j < KS / 2; ++j) {
        const int c = 4 * j + tq;
        const uint4 u0 = real0 ? *reinterpret_cast<const uint4*>(q0 + c * 8) : make_uint4(0, 0, 0, 0);
        const uint4 u1 = real1 ? *reinterpret_cast<const uint4*>(q1 + c * 8) : make_uint4(0, 0, 0, 0);
        qa[2 * j][0] = u0.x;
        qa[2 * j][1] = u1.x;
        qa[2 * j][2] = u0.y;
        qa[2 * j][3] = u1.y;
        qa[2 * j + 1][0] = u0.z;
        qa[2 * j + 1][1] = u1.z;
        qa[2 * j + 1][2] = u0.w;
        qa[2 * j + 1][3] = u1.w;
      }
    }
    const float smul = p.use_softcap ? p.cap_scale : p.scale_log2;
    const bool alibi = p.slopes != nullptr;
    const float sl0 = (alibi && real0) ? p.slopes[h0 + gq] * kLog2e : 0.0f;
    const float sl1 = (alibi && real1) ? p.slopes[h0 + gq + 8] * kLog2e : 0.0f;
    float o[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.0f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;
    // this lane's K row (B operand of the score product, n-tile 0; + 8 for n-tile 1)
    const int krow = warp * 16 + (gq >> 1) + ((gq & 1) << 2);
    // this lane's V row address for ldmatrix: matrix lane / 8 holds k-half (lane / 8) % 2
    // of n-tile 2u + lane / 16
    const int vrow = warp * 16 + ((lane >> 3) & 1) * 8 + ((lane & 7) >> 1) + ((lane & 1) << 2);
    const uint32_t sVa = smem_addr(sV);

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
        const uint8_t* kt = sK + slot * C::kTile;
        const uint32_t vt = sVa + slot * C::kTile;
        const int a = a0 + i * kRows;
        float sc[2][4];
#pragma unroll
        for (int jt = 0; jt < 2; ++jt) {
          sc[jt][0] = sc[jt][1] = sc[jt][2] = sc[jt][3] = 0.0f;
          const int r = krow + 8 * jt;
#pragma unroll
          for (int j = 0; j < KS / 2; ++j) {
            const int c = 4 * j + tq;
            const uint4 kw = *reinterpret_cast<const uint4*>(kt + (c >> 3) * C::kHalf + r * 128 +
                                                             (((c & 7) ^ (r & 7)) << 4));
            mma_16816<T>(sc[jt], qa[2 * j], kw.x, kw.y);
            mma_16816<T>(sc[jt], qa[2 * j + 1], kw.z, kw.w);
          }
        }
        // scores: modifiers, mask, running max per row
        float mt0 = -INFINITY, mt1 = -INFINITY;
#pragma unroll
        for (int jt = 0; jt < 2; ++jt) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int tok = a + warp * 16 + 8 * jt + tq + 4 * e;
            const bool vis = tok >= t0 && tok < t1;
            float x0 = sc[jt][e] * smul, x1 = sc[jt][2 + e] * smul;
            if (p.use_softcap) {
              x0 = p.cap_log2 * tanh_via_exp2(x0);
              x1 = p.cap_log2 * tanh_via_exp2(x1);
            }
            if (alibi) {
              const float dist = static_cast<float>(pos - tok);
              x0 -= sl0 * dist;
              x1 -= sl1 * dist;
            }
            sc[jt][e] = (vis && real0) ? x0 : -INFINITY;
            sc[jt][2 + e] = (vis && real1) ? x1 : -INFINITY;
            mt0 = fmaxf(mt0, sc[jt][e]);
            mt1 = fmaxf(mt1, sc[jt][2 + e]);
          }
        }
        mt0 = fmaxf(mt0, __shfl_xor_sync(0xffffffffu, mt0, 1));
        mt1 = fmaxf(mt1, __shfl_xor_sync(0xffffffffu, mt1, 1));
        mt0 = fmaxf(mt0, __shfl_xor_sync(0xffffffffu, mt0, 2));
        mt1 = fmaxf(mt1, __shfl_xor_sync(0xffffffffu, mt1, 2));
        const float mn0 = fmaxf(m0, mt0), mn1 = fmaxf(m1, mt1);
        const bool live0 = mn0 != -INFINITY, live1 = mn1 != -INFINITY;  // uniform over a row's 4 lanes
        const float al0 = live0 ? ex2(m0 - mn0) : 1.0f;
        const float al1 = live1 ? ex2(m1 - mn1) : 1.0f;
        float ps0 = 0.0f, ps1 = 0.0f;
#pragma unroll
        for (int jt = 0; jt < 2; ++jt) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            sc[jt][e] = live0 ? ex2(sc[jt][e] - mn0) : 0.0f;
            sc[jt][2 + e] = live1 ? ex2(sc[jt][2 + e] - mn1) : 0.0f;
            ps0 += sc[jt][e];
            ps1 += sc[jt][2 + e];
          }
        }
        l0 = l0 * al0 + ps0;
        l1 = l1 * al1 + ps1;
        m0 = live0 ? mn0 : m0;
        m1 = live1 ? mn1 : m1;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          o[n][0] *= al0;
          o[n][1] *= al0;
        }
        if (hi) {
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            o[n][2] *= al1;
            o[n][3] *= al1;
          }
        }
        // P as the A operand: n-tile 0 is k 0..7, n-tile 1 is k 8..15
        uint32_t pa[4];
        pa[0] = pack2<T>(sc[0][0], sc[0][1]);
        pa[1] = pack2<T>(sc[0][2], sc[0][3]);
        pa[2] = pack2<T>(sc[1][0], sc[1][1]);
        pa[3] = pack2<T>(sc[1][2], sc[1][3]);
#pragma unroll
        for (int u = 0; u < NT / 2; ++u) {
          const int cc = 2 * u + (lane >> 4);
          uint32_t vb[4];
          ldsm_x4_trans(vb, vt + (cc >> 3) * C::kHalf + vrow * 128 + (((cc & 7) ^ (vrow & 7)) << 4));
          mma_16816<T>(o[2 * u], pa, vb[0], vb[1]);
          mma_16816<T>(o[2 * u + 1], pa, vb[2], vb[3]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->empty[slot]);
    }
    // row sums over the four lanes of a row, then publish the warp's state
    // through the (now idle) ring once every consumer warp is done with it
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    asm volatile("bar.sync 1, %0;" ::"r"(kWarps * 32) : "memory");
    float* accs = reinterpret_cast<float*>(smem);  // [kWarps][G][D]
    if (real0) {
      float* row = accs + (warp * G + gq) * D + 2 * tq;
#pragma unroll
      for (int n = 0; n < NT; ++n) *reinterpret_cast<float2*>(row + 8 * n) = make_float2(o[n][0], o[n][1]);
      if (tq == 0) {
        sh->m[warp][gq] = m0;
        sh->l[warp][gq] = l0;
      }
    }
    if (real1) {
      float* row = accs + (warp * G + gq + 8) * D + 2 * tq;
#pragma unroll
      for (int n = 0; n < NT; ++n) *reinterpret_cast<float2*>(row + 8 * n) = make_float2(o[n][2], o[n][3]);
      if (tq == 0) {
        sh->m[warp][gq + 8] = m1;
        sh->l[warp][gq + 8] = l1;
      }
    }
  }
  const bool any_bad = __syncthreads_or(bad) != 0;

  const float* accs = reinterpret_cast<const float*>(smem);
  const float nan = __int_as_float(0x7fc00000);
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    const int r = idx / D, c = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sh->m[w][r]);
    float ltot = 0.0f, oc = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float x = (sh->m[w][r] == -INFINITY) ? 0.0f : ex2(sh->m[w][r] - M);
        ltot += sh->l[w][r] * x;
        oc += accs[(w * G + r) * D + c] * x;
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
    const size_t row = static_cast<size_t>(b) * p.H + h0 + r;
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
  if (tmK != nullptr && decode_on_tensor_cores(p.H, p.H_kv)) {
    static_assert(kMmaRows == 16, "decode_group_heads assumes 16 product rows");
    const int G = decode_group_heads(p.H, p.H_kv);  // query heads per CTA
    using C = MmaCfg<D>;
    auto kernel = decode_split_mma_kernel<T, D>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    dim3 g2(p.H / G * p.num_splits, p.B);
    kernel<<<g2, (kWarps + 1) * 32, C::kSmem, stream>>>(*tmK, *tmV, p, G);
  } else if (tmK != nullptr) {
    using C = TmaCfg<D>;
    static_assert(sizeof(TmaShared<D>) <= C::kShared, "decode shared block exceeds its reserve");
    auto kernel = decode_split_tma_kernel<T, D>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    kernel<<<grid, (kWarps + 1) * 32, C::kSmem, stream>>>(*tmK, *tmV, p);
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
