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
// B200 mapping. The grid is persistent (at most one CTA per SM); a CTA runs
// jobs, each one 128-row Q tile of one (batch, head), back to back with
// these warps:
//   softmax    8 warps in two parts: warps w and w + 4 share TMEM lanes
//              32 (w % 4) .. + 31 (one query row per lane); part 0 takes
//              keys 0..63 of every tile, part 1 keys 64..127. Each part runs
//              its own online softmax (its own running max, sums and O
//              accumulator), so the two never wait for each other within a
//              job; they merge their results once, at the end of the job
//   producer   TMA: each job's Q tile (two buffers, so the next job's Q
//              lands early), then K and V tiles into two rings of
//              shared-memory slots (128-byte swizzle), expect-tx
//   QK issuer  one elected thread; owns TMEM
//   PV issuer  one elected thread
// Tensor memory (512 columns x 128 lanes x 32 bit):
//   cols   0..127  S buffer 0 (fp32 scores): part p's 64 keys in columns
//                  64 p .. 64 p + 63, overwritten by its P (16-bit, two per
//                  column, or 8-bit, four per column) once it has read them;
//                  the PV products read P straight from TMEM
//   cols 128..255  S buffer 1
//   cols 256..383  O_0: part 0's accumulator (fp32, d columns)
//   cols 384..511  O_1: part 1's
// K/V tiles are numbered across the CTA's jobs; tile g uses S buffer g & 1.
// The QK thread computes S(g) as soon as K(g) has landed and the PV product
// of tile g - 2 (the last reader of the buffer, P(g - 2) included) is done;
// the PV thread computes O_p += P_p(g) V_p(g) for both parts as soon as the
// softmax has published P(g).
// Across a job boundary the next job's first scores are computed while the
// softmax warps write out the previous job's O. The two
// products are independent, so they sit in different threads: each thread
// waits on its own barriers while the other keeps the tensor pipe fed (the
// pipe queues only a couple of MMAs), and each commits once per tile. The
// next tile's scores are computed while the softmax warps work on the
// current one, so the step time is max(softmax, tensor core) rather than
// their sum.
//
// Rescaling is lazy: a part keeps its old max unless a new tile raises it
// by more than 8 (log2 units), so P stays <= 2^8 and O_p is rescaled only
// when it must be (after waiting for the previous PV product). The result is
// the same softmax (the maxima cancel in O / l): at the end of a job
// O = (a_0 O_0 + a_1 O_1) / (a_0 q_0 + a_1 q_1) with a_p = 2^(m_p - max m),
// q_p the part's sum of P as rounded.
#include "fa_internal.h"
#include "sm100_ptx.cuh"

#include <cfloat>
#include <climits>
#include <type_traits>


namespace fa {
namespace {

constexpr int BM = 128;  // query rows per Q tile
constexpr int BN = 128;  // keys per K/V tile
// Softmax warps per row (per TMEM lane quarter): two, each with its own O
// accumulator (two fill the 512 TMEM columns with the two S buffers). Warp
// roles: softmax warps 0 .. 7, then the TMA producer, the QK issuer (owns
// TMEM) and the PV issuer.
constexpr int kMaxParts = 2;
constexpr int parts_of(bool, bool) { return 2; }
constexpr int threads_of(bool cap, bool alibi) { return 32 * (4 * parts_of(cap, alibi) + 3); }
constexpr int kMaxSlots = 6;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr uint32_t kTmemCols = 512;
// Rings of completion barriers, indexed by tile number modulo kRing. No
// waiter is ever kRing tiles behind the phase it waits for: each ring
// advances only through steps that need the waiter to have passed first
// (P of a later tile, or a K/V load issued after the wait).
constexpr int kRing = 8;
constexpr uint32_t kTmemO = 256;        // O accumulator of part 0; part 1's follows
constexpr uint32_t kTmemOStride = 128;

constexpr int kBarrierBytes = 8192;  // barrier block and exchange slots
// O staging of the epilogue, after the barrier block: per softmax warp its
// 32 rows x 32 output columns (64 bytes a row)
constexpr int kStageWarpBytes = 32 * 64;
constexpr int kStageBytes = 8 * kStageWarpBytes;

// Input element types: fp16 / bf16 (products of kind::f16, P rounded to the
// input type, O written in it), or 8-bit floats (tags below: products of
// kind::f8f6f4, P rounded to the same 8-bit format, O written as bf16).
struct Fp8E4M3 {};
struct Fp8E5M2 {};

template <typename T>
struct Elem {
  using Out = T;
  static constexpr int kBytes = 2;
  static constexpr bool kFp8 = false;
  static constexpr uint32_t kFmt = 0;
};
template <>
struct Elem<Fp8E4M3> {
  using Out = __nv_bfloat16;
  static constexpr int kBytes = 1;
  static constexpr bool kFp8 = true;
  static constexpr uint32_t kFmt = 0;
};
template <>
struct Elem<Fp8E5M2> {
  using Out = __nv_bfloat16;
  static constexpr int kBytes = 1;
  static constexpr bool kFp8 = true;
  static constexpr uint32_t kFmt = 1;
};

// Shared-memory tiles: 128 rows of d elements in 128-byte swizzle chunks
// (64 elements of 16 bits or 128 of 8 bits each); a chunk of 128 rows is
// 16 KB. 8-bit V arrives transposed (d rows of 128 keys), so that both
// operands of the PV product are K-major as well.
template <typename T, int D>
struct Cfg {
  static constexpr int kRowBytes = D * Elem<T>::kBytes;
  static constexpr int kChunks = kRowBytes / 128;           // swizzle chunks per row
  static constexpr int kChunkElems = 128 / Elem<T>::kBytes;  // elements per chunk row
  static constexpr int kChunkBytes = BM * 128;               // one chunk of 128 rows
  static constexpr int kTileBytes = BM * kRowBytes;          // one Q, K or V tile
  static constexpr int kSteps = kRowBytes / 32;              // MMAs of an S product (32 bytes of d each)
  // two Q buffers, so the next job's Q lands while this one's runs
  static constexpr int kQBufs = 2;                           // active job a uses buffer a % kQBufs
  static constexpr int kSlotsK = (kTileBytes <= 16384) ? 5 : 2;  // K ring depth
  static constexpr int kSlotsV = kSlotsK;                        // V ring depth
  static constexpr int kSlots = kSlotsK + kSlotsV;
  static constexpr int kSmemBytes = 1024 + (kQBufs + kSlots) * kTileBytes + kBarrierBytes + kStageBytes;
};

struct Barriers {
  uint64_t q_full[2];   // per Q buffer (active job a uses buffer a & 1)
  uint64_t q_empty[2];  // the QK thread is done with the buffer's job
  uint64_t k_full[kMaxSlots];
  uint64_t v_full[kMaxSlots];
  // Tiles are numbered across the CTA's jobs (g). s_ready[g % kRing]: S(g)
  // is computed (commit of the QK thread), so its K slot is free too.
  // pv_done[g % kRing]: O += P(g) V(g) is complete (commit of the PV
  // thread): its V slot and P buffer are free and O is idle.
  uint64_t s_ready[kRing];
  uint64_t pv_done[kRing];
  uint64_t p_full[2];  // per P buffer
  uint64_t o_free;     // the softmax warps have read O of an active job
  uint64_t qk_idle;    // all MMAs of the QK thread complete
  uint64_t pv_idle;    // all MMAs of the PV thread complete
  uint32_t tmem_base;
  int abort;
  // per exchange parity, part and row: the partial maxima / sums of the
  // parts of a row (NaN marks a part that gave up on a timed-out wait)
  float xchg[2][kMaxParts][BM];
};

// Visible key interval [lo, hi] of query row q (empty when lo > hi).
struct RowRange {
  int lo, hi;
};

// Nq, Nk: the lengths of the query row's sequence.
__device__ __forceinline__ RowRange row_range(const FwdParams& p, int Nq, int Nk, int q) {
  const long long pos = static_cast<long long>(q) + Nk - Nq;
  long long lo = 0, hi = static_cast<long long>(Nk) - 1;
  if (p.window_left >= 0) lo = max(lo, pos - p.window_left);
  if (p.causal) hi = min(hi, pos);
  if (p.window_right >= 0) hi = min(hi, pos + p.window_right);
  RowRange r;
  r.lo = static_cast<int>(min(lo, static_cast<long long>(Nk)));
  r.hi = static_cast<int>(max(hi, -1ll));
  return r;
}

// Waits without checking the abort flag (used only to drain work in flight).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  int dummy = 0;
  mbar_wait(bar, parity, &dummy);
}

// A CTA is persistent: it runs jobs (one 128-row Q tile of one (batch,
// head) each) one after another, and every role walks the same job
// sequence. Work items pair Q tile t of a head with tile T - 1 - t (T tiles
// per head), so under a causal mask every item has the same number of K/V
// tiles; CTA c takes items c, c + gridDim.x, ... and runs the longer tile of
// each item first. Consecutive items belong to the same head, so the CTAs
// running at one time share K/V in L2.
struct Job {
  int b, h, q0, f, l;  // K/V tiles f..l
  int hk;              // K/V head of query head h
  bool has;            // at least one visible key
  int Nq, Nk;          // lengths of the job's sequence
  int qrow, krow;      // first row of the sequence in the Q and K/V maps
  int bcoord;          // batch coordinate in the maps
  long long obase;     // out row of query 0 of the sequence ((obase + q) * H + h)
  long long lbase;     // LSE index of query 0 of the sequence, head h
};

// Lengths and row offsets of sequence b; false if a variable-length table
// entry is out of its contract (the sequence is then skipped).
__device__ __forceinline__ bool seq_of(const FwdParams& p, int b, int& Nq, int& Nk, int& qrow, int& krow) {
  if (p.cu_q == nullptr) {
    Nq = p.Nq;
    Nk = p.Nk;
    qrow = krow = 0;
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

__device__ __forceinline__ Job make_job(const FwdParams& p, int b, int h, int Nq, int Nk, int qrow, int krow,
                                        int tile) {
  Job j;
  j.b = b;
  j.h = h;
  j.hk = p.H_kv == p.H ? h : h / (p.H / p.H_kv);
  j.q0 = tile * BM;
  j.Nq = Nq;
  j.Nk = Nk;
  j.qrow = qrow;
  j.krow = krow;
  const bool varlen = p.cu_q != nullptr;
  j.bcoord = varlen ? 0 : b;
  j.obase = varlen ? static_cast<long long>(qrow) : static_cast<long long>(b) * Nq;
  j.lbase = varlen ? static_cast<long long>(h) * p.total_q + qrow : (static_cast<long long>(b) * p.H + h) * Nq;
  // K/V tile range of the Q tile (rows' visible intervals are monotone in q)
  const int qz = min(j.q0 + BM - 1, Nq - 1);
  const RowRange ra = row_range(p, Nq, Nk, j.q0), rz = row_range(p, Nq, Nk, qz);
  j.has = ra.lo <= rz.hi;
  j.f = j.has ? ra.lo / BN : 0;
  j.l = j.has ? rz.hi / BN : -1;
  return j;
}

// The K/V tile a job visits u-th: f, .., l, or l, .., f with ALiBi (kRev).
// With ALiBi a row's scores grow toward its own position, so visiting the
// nearest keys first sets the running max at the first tile and the lazy
// rescale (which waits for the previous PV product) rarely fires; in key
// order it fired on nearly every tile for the steeper heads.
template <bool kRev>
__device__ __forceinline__ int tile_at(const Job& jb, int u) {
  return kRev ? jb.l - u : jb.f + u;
}

// Calls fn(job) for every job of this CTA, in order. The work items are
// numbered consecutively over the sequences (b, then head h, then pair pi;
// sequence b has H * ceil(T_b / 2) items, T_b its Q tiles), so sequences of
// different lengths leave no empty slots in the round robin; the walk over
// the sequences only moves forward.
template <typename Fn>
__device__ __forceinline__ void for_each_job(const FwdParams& p, Fn&& fn) {
  // (item counts stay below 2^31: the host checks B * H * ceil(Nq / 128))
  int b = -1;
  int base = 0, n_b = 0;  // first item of sequence b, its item count
  int Nq = 0, Nk = 0, qrow = 0, krow = 0, per_b = 1;
  for (int w = static_cast<int>(blockIdx.x);; w += static_cast<int>(gridDim.x)) {
    while (w >= base + n_b) {
      base += n_b;
      if (++b >= p.B) return;
      n_b = 0;
      if (seq_of(p, b, Nq, Nk, qrow, krow)) {
        per_b = ((Nq + BM - 1) / BM + 1) / 2;  // pairs of Q tiles per head
        n_b = p.H * per_b;
      }
    }
    const int li = w - base;
    const int h = li / per_b, pi = li % per_b;
    const int tiles = (Nq + BM - 1) / BM;
    const int t_long = tiles - 1 - pi;
    fn(make_job(p, b, h, Nq, Nk, qrow, krow, t_long));
    if (pi != t_long) fn(make_job(p, b, h, Nq, Nk, qrow, krow, pi));
  }
}

template <typename T, int D, bool kRev>
__device__ void producer(const FwdParams& p, const CUtensorMap* tmQ, const CUtensorMap* tmK, const CUtensorMap* tmV,
                         uint8_t* sQ, uint8_t* sK, uint8_t* sV, Barriers* bars) {
  using C = Cfg<T, D>;
  volatile int* abort = &bars->abort;
  const uint64_t pol_q = l2_policy_evict_first();
  const uint64_t pol_kv = l2_policy_evict_last();
  // Tile g goes to slot g % depth of its ring; the slot's previous tile
  // (g - depth) is free once the product that read it is done.
  int g = 0, a = 0;    // tiles and active jobs so far
  int nk = 0, nv = 0;  // K and V loads issued
  bool ok = true;
  auto load = [&](const CUtensorMap* map, uint8_t* ring, uint64_t* full, uint64_t* freed, int depth, int gi,
                  const Job& jb, int key_tile) -> bool {
    const int slot = gi % depth;
    if (gi >= depth && !mbar_wait(&freed[(gi - depth) % kRing], ((gi - depth) / kRing) & 1, abort)) return false;
    mbar_arrive_expect_tx(&full[slot], C::kTileBytes);
    if (Elem<T>::kFp8 && map == tmV) {
      // transposed V: box of 128 keys (the inner coordinate) x d rows
      tma_load_4d(map, &full[slot], ring + slot * C::kTileBytes, key_tile * BN, 0, jb.hk, jb.bcoord, pol_kv);
      return true;
    }
#pragma unroll
    for (int ch = 0; ch < C::kChunks; ++ch)
      tma_load_4d(map, &full[slot], ring + slot * C::kTileBytes + ch * C::kChunkBytes, ch * C::kChunkElems, jb.hk,
                  jb.krow + key_tile * BN, jb.bcoord, pol_kv);
    return true;
  };
  for_each_job(p, [&](const Job& jb) {
    if (!jb.has || !ok) return;
    const int n = jb.l - jb.f + 1;
    // Q of active job a goes to buffer a & 1 once job a - 2 is through QK
    constexpr int QB = C::kQBufs;
    if (a >= QB && !(ok = mbar_wait(&bars->q_empty[a % QB], ((a - QB) / QB) & 1, abort))) return;
    mbar_arrive_expect_tx(&bars->q_full[a % QB], C::kTileBytes);
#pragma unroll
    for (int ch = 0; ch < C::kChunks; ++ch)
      tma_load_4d(tmQ, &bars->q_full[a % QB], sQ + (a % QB) * C::kTileBytes + ch * C::kChunkBytes,
                  ch * C::kChunkElems, jb.h, jb.qrow + jb.q0, jb.bcoord, pol_q);
    auto load_k = [&](int u) {
      const bool r = load(tmK, sK, bars->k_full, bars->s_ready, C::kSlotsK, g + u, jb, tile_at<kRev>(jb, u));
      nk += r;
      return r;
    };
    auto load_v = [&](int u) {
      const bool r = load(tmV, sV, bars->v_full, bars->pv_done, C::kSlotsV, g + u, jb, tile_at<kRev>(jb, u));
      nv += r;
      return r;
    };
    // in order of need: K(0), K(1), V(0), then K(u + 2), V(u + 1)
    ok = load_k(0);
    if (ok && n > 1) ok = load_k(1);
    if (ok) ok = load_v(0);
    for (int u = 0; u + 1 < n && ok; ++u) {
      if (u + 2 < n) ok = load_k(u + 2);
      if (ok) ok = load_v(u + 1);
    }
    g += n;
    ++a;
  });
  // Every load issued must land before the CTA may exit. On the normal path
  // they all have (the MMA threads consumed them); after an abort, wait.
  for (int i = max(0, a - C::kQBufs); i < a; ++i) drain_wait(&bars->q_full[i % C::kQBufs], (i / C::kQBufs) & 1);
  for (int u = max(0, nk - C::kSlotsK); u < nk; ++u) drain_wait(&bars->k_full[u % C::kSlotsK], (u / C::kSlotsK) & 1);
  for (int u = max(0, nv - C::kSlotsV); u < nv; ++u) drain_wait(&bars->v_full[u % C::kSlotsV], (u / C::kSlotsV) & 1);
}

// S(g) = Q K_g^T into S buffer g & 1: M = 128 query rows, N = 128 keys,
// K = d in steps of 16; both operands K-major, 128-byte swizzled, 64
// elements per 16 KB chunk. Before overwriting the buffer the thread waits
// for the PV product of tile g - 2: that product waited for P(g - 2), so the
// softmax is done with S(g - 2), and once it completes P buffer g & 1 is
// free as well; the commit that publishes S(g) therefore also tells the
// softmax that it may write P(g).
template <typename T, int D>
__device__ void qk_issuer(const FwdParams& p, uint8_t* sQ, uint8_t* sK, Barriers* bars, uint32_t tmem) {
  using C = Cfg<T, D>;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr bool kFp8 = Elem<T>::kFp8;
  // a negative softmax scale is applied as -Q K^T (A-negate bit) times |scale|
  const uint32_t idesc = (kFp8 ? instr_desc_f8(Elem<T>::kFmt, BM, BN) : instr_desc_f16(kBf16, BM, BN, false)) |
                         (p.negate_scores ? (1u << 13) : 0u);
  volatile int* abort = &bars->abort;
  const uint32_t sQaddr = smem_addr(sQ), sKaddr = smem_addr(sK);
  int g = 0, a = 0;
  bool ok = true;
  for_each_job(p, [&](const Job& jb) {
    if (!jb.has || !ok) return;
    const int n = jb.l - jb.f + 1;
    if (!(ok = mbar_wait(&bars->q_full[a % C::kQBufs], (a / C::kQBufs) & 1, abort))) return;
    // Descriptors are built once per operand tile; stepping K by 16 adds a
    // byte offset to the start-address field (16-byte units, no carry:
    // shared addresses are below 2^18).
    const uint64_t qdesc = smem_desc_sw128(sQaddr + (a % C::kQBufs) * C::kTileBytes, 16, 1024);
    for (int u = 0; u < n; ++u) {
      const int gi = g + u;
      if (gi >= 2 && !(ok = mbar_wait(&bars->pv_done[(gi - 2) % kRing], ((gi - 2) / kRing) & 1, abort))) return;
      const int slot = gi % C::kSlotsK;
      if (!(ok = mbar_wait(&bars->k_full[slot], (gi / C::kSlotsK) & 1, abort))) return;
      tc_fence_after();
      const uint32_t d_t = tmem + (gi & 1) * 128;
      const uint64_t kdesc = smem_desc_sw128(sKaddr + slot * C::kTileBytes, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < C::kSteps; ++kk) {
        const uint32_t off = ((kk / 4) * C::kChunkBytes + (kk % 4) * 32) >> 4;
        if constexpr (kFp8)
          mma_ss_f8(d_t, qdesc + off, kdesc + off, idesc, kk > 0 ? 1u : 0u);
        else
          mma_ss(d_t, qdesc + off, kdesc + off, idesc, kk > 0 ? 1u : 0u);
      }
      tc_commit(&bars->s_ready[gi % kRing]);
    }
    tc_commit(&bars->q_empty[a % C::kQBufs]);
    g += n;
    ++a;
  });
  // All MMAs of this thread must be complete before TMEM is released.
  tc_commit(&bars->qk_idle);
  drain_wait(&bars->qk_idle, 0);
}

// O_p (+)= P_p(g) V_g[keys of part p] for p = 0, 1: A = P from TMEM (the
// first columns of part p's S columns in buffer g & 1), B = V tile stored
// keys x d with d contiguous (MN-major): 16 keys = 2048 bytes, the second
// 64-wide d chunk lies 16 KB further (leading byte offset); 8-bit V arrives
// transposed (K-major). The first products of a job overwrite O_0 and O_1,
// so they wait until the softmax warps have read both of the previous
// active job.
template <typename T, int D>
__device__ void pv_issuer(const FwdParams& p, uint8_t* sV, Barriers* bars, uint32_t tmem) {
  using C = Cfg<T, D>;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr bool kFp8 = Elem<T>::kFp8;
  constexpr uint32_t idesc = kFp8 ? instr_desc_f8(Elem<T>::kFmt, BM, D) : instr_desc_f16(kBf16, BM, D, true);
  volatile int* abort = &bars->abort;
  const uint32_t sVaddr = smem_addr(sV);
  int g = 0, a = 0;
  bool ok = true;
  for_each_job(p, [&](const Job& jb) {
    if (!jb.has || !ok) return;
    const int n = jb.l - jb.f + 1;
    if (a >= 1 && !(ok = mbar_wait(&bars->o_free, (a - 1) & 1, abort))) return;
    for (int u = 0; u < n; ++u) {
      const int gi = g + u;
      if (!(ok = mbar_wait(&bars->p_full[gi & 1], (gi >> 1) & 1, abort))) return;
      const int slot = gi % C::kSlotsV;
      if (!(ok = mbar_wait(&bars->v_full[slot], (gi / C::kSlotsV) & 1, abort))) return;
      tc_fence_after();
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        // part p's P lies in the first columns of its own 64 S columns;
        // O_p += P_p V[keys 64 p .. 64 p + 63]
        const uint32_t a_t = tmem + (gi & 1) * 128 + part * 64;
        const uint32_t d_t = tmem + kTmemO + part * kTmemOStride;
        if constexpr (kFp8) {
          // B = V^T tile (d rows of 128 key bytes, K-major); 32 keys per MMA
          // = 8 TMEM columns of P (four 8-bit values per column)
          const uint64_t vdesc = smem_desc_sw128(sVaddr + slot * C::kTileBytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < BN / 64; ++kk)
            mma_ts_f8(d_t, a_t + kk * 8, vdesc + ((part * 64 + kk * 32) >> 4), idesc, (u > 0 || kk > 0) ? 1u : 0u);
        } else {
          const uint64_t vdesc = smem_desc_sw128(sVaddr + slot * C::kTileBytes, C::kChunkBytes, 1024);
#pragma unroll
          for (int kk = 0; kk < BN / 32; ++kk)
            mma_ts(d_t, a_t + kk * 8, vdesc + (((part * 4 + kk) * 2048) >> 4), idesc, (u > 0 || kk > 0) ? 1u : 0u);
        }
      }
      tc_commit(&bars->pv_done[gi % kRing]);
    }
    g += n;
    ++a;
  });
  tc_commit(&bars->pv_idle);
  drain_wait(&bars->pv_idle, 0);
}

// Score transform of one element in log2 units (softcap and ALiBi paths).
template <bool kCap, bool kAlibi>
__device__ __forceinline__ float mod_score(const FwdParams& p, float x, float cap_k, float slope_l2, float dist) {
  // dist = pos - key as a float (integers below 2^24 exactly)
  const float bias = kAlibi ? -slope_l2 * fabsf(dist) : 0.0f;
  if (kCap) return softcap_fma(x, cap_k, p.cap_log2, bias);
  return fmaf(x, p.scale_log2, bias);
}

// Softmax: 8 warps, two per sub-partition. The parts warps w and w + 4 own
// the same 32 query rows (TMEM lanes 32(w % 4) ..), one row per thread, and
// each handles its own half of every 128-key tile with its own running
// state; the halves meet only in the job's epilogue, through shared memory
// under a named barrier. kCap / kAlibi select the score modifiers at compile
// time; whether a K tile needs the element mask is decided per tile for the
// whole group, so the common interior tiles run without per-element
// compares.
template <int kParts>
__device__ __forceinline__ void part_sync(int quarter) {
  // named barrier 1 + quarter, shared by the kParts warps of one lane quarter
  asm volatile("bar.sync %0, %1;" ::"r"(1 + quarter), "r"(32 * kParts) : "memory");
}

// Exchange of one value among the kParts warps of a row. All call it the
// same number of times (the k-th exchange uses slot k & 1, so a slot is
// rewritten only after every partner has passed the next barrier and hence
// read it). A part that failed passes NaN. Fills all[] with every part's
// value (own included).
template <int kParts>
__device__ __forceinline__ void part_exchange(float (&xchg)[2][kMaxParts][BM], int k, int part, int r, int quarter,
                                              float v, float (&all)[kParts]) {
  xchg[k & 1][part][r] = v;
  part_sync<kParts>(quarter);
#pragma unroll
  for (int i = 0; i < kParts; ++i) all[i] = xchg[k & 1][i][r];
}

template <typename T, int D, bool kCap, bool kAlibi>
__device__ void softmax_job(const FwdParams& p, Barriers* bars, uint32_t tmem, const Job& jb, int g, int& xk,
                            bool& alive) {
  constexpr bool kPlain = !kCap && !kAlibi;
  constexpr int kParts = parts_of(kCap, kAlibi);
  constexpr int kKeys = BN / kParts;     // keys per thread per tile
  constexpr int kChunks = kKeys / 32;    // 32-column TMEM loads of S per tile
  constexpr int kOCols = D / kParts;     // output columns per thread in the epilogue
  constexpr int kPCols = kKeys * Elem<T>::kBytes / 4;  // TMEM columns of this part's P
  static_assert(kKeys % 32 == 0 && kOCols % 32 == 0 && kParts == 2, "part sizes");
  using Out = typename Elem<T>::Out;
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int part = warp >> 2;
  const int r = quarter * 32 + lane;  // row of the tile == TMEM lane
  const int h = jb.h, q0 = jb.q0, f = jb.f, l = jb.l;
  const int q = q0 + r;
  const bool row_ok = q < jb.Nq;
  const RowRange rr = row_range(p, jb.Nq, jb.Nk, row_ok ? q : jb.Nq - 1);
  // tile-level bounds: a K tile needs no mask when every row of the tile
  // sees all of it (rows' intervals are monotone in q)
  const int qz = min(q0 + BM - 1, jb.Nq - 1);
  const RowRange first_row = row_range(p, jb.Nq, jb.Nk, q0), last_row = row_range(p, jb.Nq, jb.Nk, qz);
  const int pos = q + jb.Nk - jb.Nq;
  const uint32_t lane_sel = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tO = tmem + lane_sel + kTmemO + part * kTmemOStride;  // this part's O accumulator
  const float slope_l2 = kAlibi ? p.slopes[h] * kLog2e : 0.0f;
  const float cap_k = p.cap_scale * 2.8853900817779268f;  // 2 log2(e) / softcap * |scale|
  const float sl2 = p.scale_log2;  // >= 0 (a negative scale is folded into the MMA)
  const uint64_t mul2 = kPlain ? f2_pack(sl2, sl2) : f2_pack(1.0f, 1.0f);
  const float nan = __int_as_float(0x7fc00000);

  // This part's own online softmax over its kKeys keys of every tile: its
  // own running max, sums and O accumulator, merged with the other part's
  // once, at the end of the job.
  float m = -INFINITY;  // running max of this part's keys (log2 units)
  float lsum = 0.0f;    // running sum of exp2(t - m) (for LSE)
  float qsum = 0.0f;    // the same sum of P as rounded for the PV product (for O)
  bool ok = alive;      // after a failure in an earlier job, only fill
  const int n = jb.has ? l - f + 1 : 0;
  const int n_run = ok ? n : 0;
  for (int it = 0; it < n_run; ++it) {
    const int j = tile_at<kAlibi>(jb, it);
    const int gi = g + it;  // tile number across the CTA's jobs
    const uint32_t tS = tmem + lane_sel + (gi & 1) * 128 + part * 64;  // this part's S, then P, columns
    ok = mbar_wait(&bars->s_ready[gi % kRing], (gi / kRing) & 1, abort);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    uint32_t s[kChunks][32];
    const int key0 = j * BN + part * kKeys;
    // distance of the tile's first key from the row's position; element e of
    // the tile is dpos - e away (ALiBi)
    const float dpos = kAlibi ? static_cast<float>(pos - key0) : 0.0f;
    const bool masked = j * BN < last_row.lo || j * BN + BN - 1 > first_row.hi;  // uniform over the tile
    // key visible iff (unsigned)(key - mlo) <= mspan (an empty interval:
    // mlo = -1, mspan = 0, and no key >= 0 passes)
    const bool row_has = rr.lo <= rr.hi;
    const int mlo = row_has ? rr.lo : -1;
    const unsigned mspan = row_has ? static_cast<unsigned>(rr.hi - rr.lo) : 0u;
    tc_fence_after();
#pragma unroll
    for (int c = 0; c < kChunks; ++c) tmem_ld32(tS + 32 * c, s[c]);
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < kChunks; ++c) reg_fence(s[c]);
    // pass 1: transform (modifier paths), mask and this part's max
    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      if (!kPlain || masked) {
        // (written as a lambda: this form of the loop measured 397 against
        // 375 TFLOP/s for ALiBi + softcap, the same arithmetic inline)
        auto transform = [&]() {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            float x = __uint_as_float(s[c][e]);
            const int key = key0 + 32 * c + e;
            if constexpr (!kPlain)
              x = mod_score<kCap, kAlibi>(p, x, cap_k, slope_l2, dpos - static_cast<float>(32 * c + e));
            if (masked) x = (static_cast<unsigned>(key - mlo) <= mspan) ? x : -INFINITY;
            s[c][e] = __float_as_uint(x);
          }
        };
        transform();
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
    float mt = fmaxf(fmax3(mx[0], mx[1], mx[2]), mx[3]);
    // plain path: the max was taken over raw scores; scale after (sl2 >= 0)
    if (kPlain) mt = (mt == -INFINITY) ? -INFINITY : mt * sl2;

    // lazy max update
    const float m_new = fmaxf(m, mt);
    float alpha = 1.0f;
    bool rescale = false;
    if (m == -INFINITY) {
      m = m_new;  // nothing accumulated yet for this part (its O is 0, l is 0)
    } else if (m_new > m + kRescaleThreshold) {
      alpha = ex2(m - m_new);
      m = m_new;
      rescale = true;
    }
    lsum *= alpha;
    qsum *= alpha;
    const float m_eff = (m == -INFINITY) ? 0.0f : m;
    // pass 2: P = exp2(t - m) over this part's own S columns (read above);
    // pairs of elements go through packed fp32x2 FMA (scale, subtract max)
    // and add. O is normalised by the sum of P exactly as the PV product
    // sees it (the rounded values), so rounding P perturbs the weights of a
    // convex combination of V rows rather than its total; LSE takes the sum
    // of the unrounded values.
    const uint64_t m2 = f2_pack(-m_eff, -m_eff);
    uint64_t rsum2[4] = {0, 0, 0, 0};  // independent packed partial sums (0 bits = +0.0f)
    uint64_t qsum2[2] = {0, 0};        // the same, of the rounded P
    auto pass2 = [&](auto masked_tag) {
      constexpr bool kMaskedTile = decltype(masked_tag)::value;
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float x0 = __uint_as_float(s[c][2 * e]);
          const float x1 = __uint_as_float(s[c][2 * e + 1]);
          const uint64_t a2 = f2_fma(f2_pack(x0, x1), mul2, m2);
          // every exponential on the MUFU (ex2.approx): the issue slots, not
          // the MUFU, bound this loop, and a polynomial on the FMA pipe would
          // cost about five times the issue slots
          float a0, a1;
          f2_unpack(a2, a0, a1);
          float p0 = ex2(a0), p1 = ex2(a1);
          if (kMaskedTile) {
            // masked entries hold -inf, and a zero scale makes -inf * 0 a
            // NaN: select them out
            p0 = (x0 == -INFINITY) ? 0.0f : p0;
            p1 = (x1 == -INFINITY) ? 0.0f : p1;
          }
          rsum2[e & 3] = f2_add(rsum2[e & 3], f2_pack(p0, p1));
          if constexpr (Elem<T>::kFp8) {
            // P <= 2^8 fits the 8-bit format's range; the pair's 16 bits
            // are merged four keys to a column below
            pk[e] = pack2_f8<Elem<T>::kFmt>(p0, p1);
            qsum2[e & 1] = f2_add(qsum2[e & 1], widen2_f8<Elem<T>::kFmt>(pk[e]));
          } else {
            pk[e] = pack2<T>(p0, p1);
            qsum2[e & 1] = f2_add(qsum2[e & 1], widen2<T>(pk[e]));
          }
        }
        if constexpr (Elem<T>::kFp8) {
          uint32_t pk4[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) pk4[i] = pk[2 * i] | (pk[2 * i + 1] << 16);
          tmem_st8(tS + 8 * c, pk4);
        } else {
          tmem_st16(tS + 16 * c, pk);
        }
      }
    };
    // masked entries hold -inf, whose exponential is 0 unless a zero scale
    // turns -inf * 0 into a NaN (plain path): only then select them out
    if (kPlain && masked && sl2 == 0.0f)
      pass2(std::true_type{});
    else
      pass2(std::false_type{});
    float r0, r1, r2, r3, u0, u1;
    f2_unpack(f2_add(rsum2[0], rsum2[1]), r0, r1);
    f2_unpack(f2_add(rsum2[2], rsum2[3]), r2, r3);
    f2_unpack(f2_add(qsum2[0], qsum2[1]), u0, u1);
    lsum += (r0 + r1) + (r2 + r3);
    qsum += u0 + u1;
    if (__any_sync(0xffffffffu, rescale)) {
      // this part's O must be idle: wait for the product of the previous
      // tile (the only one that can still be running)
      if (it > 0) {
        ok = mbar_wait(&bars->pv_done[(gi - 1) % kRing], ((gi - 1) / kRing) & 1, abort);
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
      }
      if (ok) {
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
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->p_full[gi & 1]);
    if (!ok) break;
  }
  if (ok && n_run > 0) {
    ok = mbar_wait(&bars->pv_done[(g + n - 1) % kRing], ((g + n - 1) / kRing) & 1, abort);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
  }
  // Merge the parts of the row (three exchanges, made by both parts of
  // every job that had keys, while no earlier job failed): M = max m_p,
  // a_p = 2^(m_p - M); O = sum a_p O_p / sum a_p q_p, LSE from sum a_p l_p.
  float a_self = 0.0f, a_other = 0.0f, ltot = 0.0f, qtot = 0.0f;
  if (alive && n > 0) {
    float mm[kParts], ll[kParts], qq[kParts];
    part_exchange(bars->xchg, xk++, part, r, quarter, ok ? m : nan, mm);
    part_exchange(bars->xchg, xk++, part, r, quarter, ok ? lsum : nan, ll);
    part_exchange(bars->xchg, xk++, part, r, quarter, ok ? qsum : nan, qq);
    float M = -INFINITY;
    bool none_nan = true;
#pragma unroll
    for (int i = 0; i < kParts; ++i) {
      none_nan = none_nan && ll[i] == ll[i] && qq[i] == qq[i] && !(mm[i] != mm[i]);
      M = fmaxf(M, mm[i]);
    }
    ok = ok && none_nan;
    if (ok) {
#pragma unroll
      for (int i = 0; i < kParts; ++i) {
        const float ai = (mm[i] == -INFINITY) ? 0.0f : ex2(mm[i] - M);
        ltot += ai * ll[i];
        qtot += ai * qq[i];
        if (i == part) a_self = ai;
        else a_other = ai;
      }
      m = M;
    }
  }

  // epilogue: this part's kOCols output columns of the row, from both O
  // accumulators: (a_0 O_0 + a_1 O_1) / (a_0 q_0 + a_1 q_1), as Out;
  // LSE = (M + log2 l) ln 2
  Out* orow = reinterpret_cast<Out*>(p.out) + ((jb.obase + (row_ok ? q : 0)) * p.H + h) * D + part * kOCols;
  // (out_scale: the dequantisation factor of 8-bit V, else 1)
  const float inv = qtot > 0.0f ? p.out_scale / qtot : 0.0f;
  const uint32_t tO_self = tO + part * kOCols;                                  // own O, own columns
  const uint32_t tO_other = tmem + lane_sel + kTmemO + (1 - part) * kTmemOStride + part * kOCols;
  if (ok && n > 0) {
    // Each row's 32 columns of a round go through this warp's staging tile
    // (16-byte chunk c of row r at chunk c ^ ((r >> 1) & 3), so that both
    // the row-wise writes and the chunk-wise reads hit every bank once),
    // and leave as stores of 8 rows x 64 bytes; a thread storing its own
    // row would touch 32 separate lines per instruction.
    uint8_t* stage = reinterpret_cast<uint8_t*>(bars) + kBarrierBytes + warp * kStageWarpBytes;
    Out* ocol = reinterpret_cast<Out*>(p.out) + static_cast<long long>(h) * D + part * kOCols;
#pragma unroll
    for (int cc = 0; cc < kOCols / 32; ++cc) {
      uint32_t o[32], o2[32];
      tmem_ld32(tO_self + 32 * cc, o);
      tmem_ld32(tO_other + 32 * cc, o2);
      tmem_wait_ld();
      reg_fence(o);
      reg_fence(o2);
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float v0 = (a_self * __uint_as_float(o[2 * e]) + a_other * __uint_as_float(o2[2 * e])) * inv;
        const float v1 = (a_self * __uint_as_float(o[2 * e + 1]) + a_other * __uint_as_float(o2[2 * e + 1])) * inv;
        pk[e] = pack2<Out>(v0, v1);
      }
#pragma unroll
      for (int v = 0; v < 4; ++v)
        *reinterpret_cast<uint4*>(stage + lane * 64 + ((v ^ ((lane >> 1) & 3)) * 16)) =
            make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int rl = 8 * i + (lane >> 2), ch = lane & 3;  // row of the warp's 32, 16-byte chunk
        const uint4 val = *reinterpret_cast<const uint4*>(stage + rl * 64 + ((ch ^ ((rl >> 1) & 3)) * 16));
        const int qr = q0 + quarter * 32 + rl;
        if (qr < jb.Nq)
          *reinterpret_cast<uint4*>(ocol + (jb.obase + qr) * p.H * D + 32 * cc + 8 * ch) = val;
      }
      __syncwarp();
    }
    // both O accumulators have been read (by both parts, which each arrive
    // here): the next job's first PV product may overwrite them
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->o_free);
  } else if (row_ok) {
    const float fill = ok ? 0.0f : nan;
    const uint32_t w = pack2<Out>(fill, fill);
    uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
    for (int v = 0; v < kOCols / 8; ++v) dst[v] = make_uint4(w, w, w, w);
  }
  if (row_ok && part == 0) {
    float lse_v;
    if (!ok) lse_v = nan;
    else if (ltot > 0.0f) lse_v = (m + lg2(ltot)) * kLn2;
    else lse_v = -INFINITY;
    p.lse[jb.lbase + q] = lse_v;
  }
  alive = alive && ok;
}

template <typename T, int D, bool kCap, bool kAlibi>
__device__ void softmax_group(const FwdParams& p, Barriers* bars, uint32_t tmem) {
  int g = 0, xk = 0;
  bool alive = true;
  for_each_job(p, [&](const Job& jb) {
    softmax_job<T, D, kCap, kAlibi>(p, bars, tmem, jb, g, xk, alive);
    if (jb.has) g += jb.l - jb.f + 1;
  });
}

template <typename T, int D, bool kCap, bool kAlibi>
__global__ void __launch_bounds__(threads_of(kCap, kAlibi), 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = Cfg<T, D>;
  constexpr int kSoftmaxWarps = 4 * parts_of(kCap, kAlibi);
  constexpr int kProducerWarp = kSoftmaxWarps;
  constexpr int kQkWarp = kSoftmaxWarps + 1;
  constexpr int kPvWarp = kSoftmaxWarps + 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;  // two Q buffers
  uint8_t* sK = smem + C::kQBufs * C::kTileBytes;
  uint8_t* sV = sK + C::kSlotsK * C::kTileBytes;
  Barriers* bars = reinterpret_cast<Barriers*>(sV + C::kSlotsV * C::kTileBytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->q_full[i], 1);
      mbar_init(&bars->q_empty[i], 1);
      mbar_init(&bars->p_full[i], kSoftmaxWarps);
    }
    for (int i = 0; i < C::kSlotsK; ++i) mbar_init(&bars->k_full[i], 1);
    for (int i = 0; i < C::kSlotsV; ++i) mbar_init(&bars->v_full[i], 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&bars->s_ready[i], 1);
      mbar_init(&bars->pv_done[i], 1);
    }
    mbar_init(&bars->o_free, kSoftmaxWarps);
    mbar_init(&bars->qk_idle, 1);
    mbar_init(&bars->pv_idle, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kQkWarp) {
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

  if (warp < kSoftmaxWarps) {
    softmax_group<T, D, kCap, kAlibi>(p, bars, tmem);
  } else if (warp == kProducerWarp) {
    if (lane == 0) producer<T, D, kAlibi>(p, &tmQ, &tmK, &tmV, sQ, sK, sV, bars);
  } else if (warp == kQkWarp) {
    if (lane == 0) qk_issuer<T, D>(p, sQ, sK, bars, tmem);
  } else if (warp == kPvWarp) {
    if (lane == 0) pv_issuer<T, D>(p, sV, bars, tmem);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kQkWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <typename T, int D, bool kCap, bool kAlibi>
cudaError_t launch(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV, const FwdParams& p,
                   cudaStream_t stream) {
  using C = Cfg<T, D>;
  static_assert(sizeof(Barriers) <= kBarrierBytes, "barrier block exceeds its reserve");
  static_assert(C::kSmemBytes <= 232448, "shared memory budget exceeded");
  static_assert(C::kSlotsK <= kMaxSlots && C::kSlotsV <= kMaxSlots, "too many K/V slots");
  auto kernel = fwd_kernel<T, D, kCap, kAlibi>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  // persistent: one CTA per SM at most (one fits per SM: shared memory, TMEM)
  static int sm_count[64];
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (sm_count[dev] == 0) {
    e = cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  const long long items = static_cast<long long>(p.B) * p.H * ((p.num_tiles + 1) / 2);
  dim3 grid(static_cast<unsigned>(items < sm_count[dev] ? items : sm_count[dev]));
  kernel<<<grid, threads_of(kCap, kAlibi), C::kSmemBytes, stream>>>(tmQ, tmK, tmV, p);
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

cudaError_t launch_fwd_fp8(int fmt, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmVt,
                           const FwdParams& p, cudaStream_t stream) {
  return fmt == 0 ? launch_mods<Fp8E4M3, 128>(tmQ, tmK, tmVt, p, stream)
                  : launch_mods<Fp8E5M2, 128>(tmQ, tmK, tmVt, p, stream);
}

namespace {

// V [B, Nk, H_kv, 128] (8-bit) -> V^T [B, H_kv, 128, Nk_pad], keys Nk ..
// Nk_pad - 1 zero-filled: one CTA per (64-key block, head, batch) stages the
// block in shared memory, 16-byte loads and stores.
__global__ void __launch_bounds__(256) v_transpose_kernel(const uint8_t* __restrict__ v, uint8_t* __restrict__ vt,
                                                          int Nk, int H_kv, int Nk_pad) {
  constexpr int D = 128;
  constexpr int kPitch = D + 16;  // bytes per staged key row
  __shared__ __align__(16) uint8_t tile[64 * kPitch];
  const int k0 = static_cast<int>(blockIdx.x) * 64;
  const int hk = static_cast<int>(blockIdx.y);
  const long long b = blockIdx.z;
  for (int idx = threadIdx.x; idx < 64 * (D / 16); idx += blockDim.x) {
    const int key = idx / (D / 16), c16 = idx % (D / 16);
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (k0 + key < Nk)
      val = *reinterpret_cast<const uint4*>(v + ((b * Nk + k0 + key) * H_kv + hk) * D + 16 * c16);
    *reinterpret_cast<uint4*>(tile + key * kPitch + 16 * c16) = val;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < D * 4; idx += blockDim.x) {
    const int c = idx / 4, part = idx % 4;
    if (k0 + 16 * part >= Nk_pad) continue;
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int kk = 16 * part + 4 * i;
      w[i] = static_cast<uint32_t>(tile[kk * kPitch + c]) | (static_cast<uint32_t>(tile[(kk + 1) * kPitch + c]) << 8) |
             (static_cast<uint32_t>(tile[(kk + 2) * kPitch + c]) << 16) |
             (static_cast<uint32_t>(tile[(kk + 3) * kPitch + c]) << 24);
    }
    *reinterpret_cast<uint4*>(vt + ((b * H_kv + hk) * D + c) * static_cast<long long>(Nk_pad) + k0 + 16 * part) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace

cudaError_t launch_v_transpose(const void* v, void* vt, int B, int Nk, int H_kv, int Nk_pad, cudaStream_t stream) {
  if (B == 0 || H_kv == 0 || Nk_pad == 0) return cudaSuccess;
  dim3 grid(static_cast<unsigned>((Nk_pad + 63) / 64), static_cast<unsigned>(H_kv), static_cast<unsigned>(B));
  v_transpose_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint8_t*>(v), static_cast<uint8_t*>(vt), Nk, H_kv,
                                               Nk_pad);
  return cudaGetLastError();
}

}  // namespace fa

