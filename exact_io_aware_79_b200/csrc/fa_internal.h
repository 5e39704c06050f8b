// fa_internal.h -- parameter blocks and launchers shared between the C-ABI
// layer (fa_api.cu) and the kernel translation units. Not part of the ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime_api.h>

namespace fa {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Forward: a persistent grid; a job is one 128-row query tile of one (b, h).
// Fixed length: Q/out [B, Nq, H, d], K/V [B, Nk, H, d], LSE [B, H, Nq].
// Variable length (cu_q != nullptr): Q/out [total_q, H, d], K/V
// [total_k, H, d], LSE [H, total_q]; sequence b owns rows
// cu_q[b] .. cu_q[b+1]-1 and cu_k[b] .. cu_k[b+1]-1, and Nq, Nk are the
// maximum lengths.
struct FwdParams {
  void* out;
  float* lse;
  const float* slopes;  // [H] or nullptr
  const int* cu_q;      // [B + 1] or nullptr (fixed length)
  const int* cu_k;      // [B + 1] or nullptr
  int total_q, total_k; // variable length: rows of Q and K/V
  int B, H, Nq, Nk;
  int H_kv;             // K/V heads (H % H_kv == 0); query head h reads K/V head h / (H / H_kv)
  int num_tiles;        // ceil(Nq / 128)
  int causal;
  int window_left, window_right;  // -1 = unbounded
  int use_softcap;
  int negate_scores;  // 1 when scale < 0: S = -Q K^T and the scales below use |scale|
  float scale_log2;  // |scale| * log2(e)                (no softcap)
  float cap_scale;   // scale / softcap                   (softcap)
  float cap_log2;    // softcap * log2(e)                 (softcap)
  float out_scale;   // O factor: the dequantisation factor of 8-bit V, else 1
};

// Paged decode, split kernel + merge kernel.
struct DecodeParams {
  const void* q;        // [B, 1, H, d]
  const void* k_cache;  // [num_pages, page_size, H, d]
  const void* v_cache;
  const int* block_table;    // [B, max_blocks]
  const int* cache_seqlens;  // [B]
  void* out;                 // [B, 1, H, d]   (num_splits == 1)
  float* lse;                // [B, H, 1]      (num_splits == 1)
  float* o_part;             // [S, B, H, d]   (num_splits > 1)
  float* lse_part;           // [S, B, H]      (num_splits > 1)
  const float* slopes;       // [H] or nullptr
  int B, H, num_pages, page_size, max_blocks, num_splits;
  int H_kv;                  // cache heads; query head h reads cache head h / (H / H_kv)
  int window_left;
  int use_softcap;
  float scale_log2, cap_scale, cap_log2;
};

// Launches the forward kernel for (dtype, d); the tensor maps describe Q, K, V
// as 4-D tensors (d, H, N, B) with a (64, 1, 128, 1) box and 128-byte swizzle.
cudaError_t launch_fwd(bool bf16, int d, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                       const FwdParams& p, cudaStream_t stream);

// The forward on 8-bit inputs (fmt 0 = E4M3, 1 = E5M2; d = 128; output bf16):
// Q and K maps (d, H, N, B) with a (128, 1, 128, 1) box of bytes, 128-byte
// swizzle; tmVt: the transposed V written by launch_v_transpose, a map
// (Nk_pad, d, H_kv, B) with a (128, 128, 1, 1) box.
cudaError_t launch_fwd_fp8(int fmt, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmVt,
                           const FwdParams& p, cudaStream_t stream);

// V [B, Nk, H_kv, 128] (8-bit) -> V^T [B, H_kv, 128, Nk_pad] with keys
// Nk .. Nk_pad - 1 set to zero (Nk_pad a multiple of 16).
cudaError_t launch_v_transpose(const void* v, void* vt, int B, int Nk, int H_kv, int Nk_pad, cudaStream_t stream);

// Grouped-query caches (two or more query heads per cache head) take the
// tensor-core split kernel; it wants 128-byte-swizzled (64, 1, 64, 1) boxes.
inline bool decode_on_tensor_cores(int H, int H_kv) { return H_kv > 0 && H / H_kv >= 2; }

// Query heads one grouped-query decode CTA serves: the largest divisor of the
// group H / H_kv that fits the 16 rows of its products.
inline int decode_group_heads(int H, int H_kv) {
  const int group = H / H_kv;
  for (int g = 16; g > 1; --g)
    if (group % g == 0) return g;
  return 1;
}

// tmK/tmV: 4-D maps (d, H, page_size, num_pages) of the caches for the
// TMA-staged split kernels (page_size % 64 == 0): a (d, 1, 64, 1) box without
// swizzle, or (64, 1, 64, 1) boxes with 128-byte swizzle when
// decode_on_tensor_cores(H, H_kv); nullptr for the direct-load split kernel.
cudaError_t launch_decode(bool bf16, int d, const DecodeParams& p, const CUtensorMap* tmK, const CUtensorMap* tmV,
                          cudaStream_t stream);

// Backward: dQ, dK, dV of L = sum(dO * O) from Q, K, V, O, LSE, dO.
struct BwdParams {
  const void* out;    // [B, Nq, H, d]
  const void* dout;   // [B, Nq, H, d]
  const float* lse;   // [B, H, Nq] (natural log, the forward's)
  float* dvec;        // [B, H, Nq] workspace: D_i = sum_c dO_ic O_ic
  float* dq_acc;      // [B, Nq, H, d] workspace: unscaled dQ in fp32
  int* job_counter;   // workspace: next job of the tensor-core kernels, [0] key blocks, [1] dQ tiles
                      // (zeroed by the row-dot kernel)
  void* dq;           // [B, Nq, H, d]
  void* dk;           // [B, Nk, H_kv, d]
  void* dv;           // [B, Nk, H_kv, d]
  const float* slopes;  // [H] or nullptr
  const int* cu_q;      // [B + 1] row offsets (packed sequences) or nullptr (fixed length)
  const int* cu_k;      // [B + 1] or nullptr
  int total_q, total_k; // packed: rows of q and of k
  long long dq_tok;     // elements from one token's dq row to the next (H * d, or 3 * H * d in a packed dqkv)
  long long dkv_tok;    // the same for dk, dv (H_kv * d, or 3 * H * d)
  int B, H, H_kv, Nq, Nk;  // packed: Nq, Nk bound the sequence lengths
  int causal, window_left, window_right;
  int use_softcap;
  int deterministic;  // 1: dQ summed in a fixed order (no atomics)
  float scale;       // softmax scale (dQ, dK factor)
  float scale_log2;  // scale * log2(e)            (no softcap)
  float cap_scale;   // scale / softcap             (softcap)
  float cap_log2;    // softcap * log2(e)           (softcap)
};

// tmQ/tmO: (d, H, Nq, B) maps of Q and dO, tmK/tmV: (d, H_kv, Nk, B) maps of
// K and V, all with (64, 1, 64, 1) boxes and 128-byte swizzle; tmDQ: the fp32
// dQ accumulator as (d, H, Nq, B) with (32, 1, 64, 1) boxes, 128-byte swizzle.
cudaError_t launch_bwd(bool bf16, int d, const BwdParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                       const CUtensorMap& tmV, const CUtensorMap& tmO, const CUtensorMap& tmDQ,
                       cudaStream_t stream);

// The key-block kernel on the tensor cores (d = 64 or 128; dK, dV, and the dQ
// partials added into p.dq_acc by TMA reduce-add through tmDQ unless
// p.deterministic): persistent CTAs claim jobs
// from *p.job_counter, which must be zero at launch. The maps as for
// launch_bwd.
cudaError_t launch_bwd_tc(bool bf16, int d, const BwdParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                          const CUtensorMap& tmV, const CUtensorMap& tmO, const CUtensorMap& tmDQ,
                          cudaStream_t stream);

// The deterministic mode's dQ pass (d = 64 or 128) on the tensor cores: dq =
// scale * sum over key blocks (fixed order) of dS K, written to p.dq;
// persistent CTAs claim 128-query tiles from p.job_counter[1], which must be
// zero at launch. The maps as for launch_bwd.
cudaError_t launch_bwd_dq_tc(bool bf16, int d, const BwdParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                             const CUtensorMap& tmV, const CUtensorMap& tmO, cudaStream_t stream);

// Writes n_new new tokens per sequence into the paged caches at positions
// cache_seqlens[b] .. cache_seqlens[b] + n_new - 1.
struct AppendParams {
  const void* k_new;  // [B, n_new, H_kv, d]
  const void* v_new;
  void* k_cache;      // [num_pages, page_size, H_kv, d]
  void* v_cache;
  const int* block_table;    // [B, max_blocks]
  const int* cache_seqlens;  // [B]
  int B, n_new, H_kv, d, num_pages, page_size, max_blocks;
};

cudaError_t launch_append(const AppendParams& p, cudaStream_t stream);

}  // namespace fa
