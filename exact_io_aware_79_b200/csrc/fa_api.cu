// fa_api.cu -- the C ABI declared in include/fa.h: argument validation,
// device check, TMA tensor-map encoding, split-count resolution and launches.
#include "fa.h"
#include "fa_internal.h"

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace {

constexpr int kNumSms = 148;           // B200; only steers the automatic split count
constexpr long long kMaxSeq = 1 << 28; // Nq, Nk limit of fa_fwd
constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 0 = unknown, 1 = sm_100, 2 = other
std::atomic<int> g_device_kind[kMaxDevices];

fa_status check_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return FA_ERR_DEVICE;
  }
  if (dev < kMaxDevices) {
    const int k = g_device_kind[dev].load(std::memory_order_relaxed);
    if (k == 1) return FA_OK;
    if (k == 2) return FA_ERR_DEVICE;
  }
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_DEVICE;
  }
  const bool ok = major == 10 && minor == 0;
  if (dev < kMaxDevices) g_device_kind[dev].store(ok ? 1 : 2, std::memory_order_relaxed);
  return ok ? FA_OK : FA_ERR_DEVICE;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// [B, N, H, d] 16-bit tensor as a 4-D map (d, H, N, B), box (64, 1, rows, 1),
// 128-byte swizzle; rows past N read as zero. tok: elements from one token
// to the next (H * d when contiguous; 3 * H * d inside a packed QKV tensor).
bool make_map(CUtensorMap* map, const void* base, bool bf16, int B, int N, int H, int d, long long tok = 0,
              int rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t n = static_cast<cuuint64_t>(N > 0 ? N : 1);
  const cuuint64_t t = static_cast<cuuint64_t>(tok > 0 ? tok : static_cast<long long>(H) * d);
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), n, static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2, t * 2, n * t * 2};
  cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(rows), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
                         const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Paged cache [num_pages, page_size, H, d] as a 4-D map (d, H, page_size,
// num_pages). One box is a 64-token slice of one page for one head: all d
// columns without swizzle, or (swizzled) 64 columns with 128-byte swizzle.
bool make_cache_map(CUtensorMap* map, const void* base, bool bf16, int num_pages, int page_size, int H, int d,
                    bool swizzled) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(page_size), static_cast<cuuint64_t>(num_pages)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2,
                           static_cast<cuuint64_t>(page_size) * H * d * 2};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(swizzled ? 64 : d), 1, 64, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
                         const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swizzled ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// fp32 [B, N, H, d] tensor as a 4-D map (d, H, N, B) with (32, 1, 64, 1)
// boxes and 128-byte swizzle (the backward's dQ accumulator).
// 8-bit [B, N, H, d] tensor (d = 128): a (128, 1, 128, 1) box of bytes, one
// 128-byte swizzle row per token.
bool make_map_u8(CUtensorMap* map, const void* base, int B, int N, int H, int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t n = static_cast<cuuint64_t>(N > 0 ? N : 1);
  const cuuint64_t t = static_cast<cuuint64_t>(H) * d;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), n, static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d), t, n * t};
  cuuint32_t box[4] = {128, 1, 128, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Transposed 8-bit V [B, H_kv, d, Nk_pad]: a (128, 128, 1, 1) box (128 keys of
// 128 rows of d), 128-byte swizzle.
bool make_map_vt(CUtensorMap* map, void* base, int B, int H_kv, int d, int Nk_pad) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t np = static_cast<cuuint64_t>(Nk_pad);
  cuuint64_t dims[4] = {np, static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H_kv), static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {np, np * d, np * d * H_kv};
  cuuint32_t box[4] = {128, 128, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, base, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Keys of the transposed 8-bit V rounded up to 16 (16-byte rows for TMA).
long long fp8_keys_padded(int Nk) { return (static_cast<long long>(Nk) + 15) / 16 * 16; }

bool make_map_f32(CUtensorMap* map, void* base, int B, int N, int H, int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t t = static_cast<cuuint64_t>(H) * d;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 4, t * 4, static_cast<cuuint64_t>(N) * t * 4};
  cuuint32_t box[4] = {32, 1, 64, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool finite(float x) { return std::isfinite(x); }

// Automatic split count: enough splits that a split of the longest possible
// sequence holds at most ~2048 keys, and, for small batches, enough CTAs to
// cover the GPU several times (but never splits shorter than 256 keys).
int auto_splits(int B, int H, long long max_len) {
  const long long units = static_cast<long long>(B) * H;
  long long s = (max_len + 2047) / 2048;
  const long long fill = (4LL * kNumSms + units - 1) / units;
  const long long min_chunk = (max_len + 255) / 256;
  s = std::max(s, std::min(fill, min_chunk));
  s = std::max(1LL, std::min(s, static_cast<long long>(FA_MAX_SPLITS)));
  return static_cast<int>(s);
}

// Split count a decode launch uses. An explicit num_splits is used as
// given. The automatic count is auto_splits; a grouped-query cache on the
// tensor-core kernel (one CTA serves G query heads and streams their cache
// head once) aims instead at the CTAs launched: about 2048 * G keys a split
// and enough CTAs to fill the GPU, never above the one-head count, so a
// workspace sized by fa_kvcache_workspace_size always holds the partials.
// Returns -1 for invalid sizes.
int launch_splits(int B, int H, int H_kv, int d, int max_blocks, int page_size, int num_splits) {
  const int S = fa_kvcache_num_splits(B, H, d, max_blocks, page_size, num_splits);
  if (S < 0 || H_kv < 1 || H_kv > H || H % H_kv != 0) return -1;
  if (num_splits != 0 || S <= 1 || page_size % 64 != 0 || !fa::decode_on_tensor_cores(H, H_kv)) return S;
  const long long G = fa::decode_group_heads(H, H_kv);
  const long long max_len = static_cast<long long>(max_blocks) * page_size;
  const long long units = static_cast<long long>(B) * (H / G);
  long long s = ((max_len + 2047) / 2048 + G - 1) / G;
  s = std::max(s, std::min((4LL * kNumSms + units - 1) / units, (max_len + 255) / 256));
  return static_cast<int>(std::max(1LL, std::min(s, static_cast<long long>(S))));
}

// Workspace bytes of S split partials: O_part [S, B, H, d] fp32, padded to
// 256 bytes, then LSE_part [S, B, H] fp32.
size_t partial_bytes(int S, int B, int H, int d) {
  if (S <= 1) return 0;
  const size_t rows = static_cast<size_t>(S) * B * H;
  const size_t o_bytes = (rows * d * sizeof(float) + 255) & ~size_t(255);
  return o_bytes + rows * sizeof(float);
}

bool kvcache_sizes_ok(int B, int H, int d, int max_blocks, int page_size) {
  if (B < 0 || H < 1 || max_blocks < 1 || page_size < 1) return false;
  if (d != 64 && d != 128) return false;
  if (static_cast<long long>(max_blocks) * page_size >= (1LL << 31)) return false;
  if (static_cast<long long>(B) * H * FA_MAX_SPLITS >= (1LL << 31)) return false;
  if (B > 65535) return false;
  return true;
}

}  // namespace

namespace {

// Shared body of fa_fwd and fa_fwd_varlen. Fixed length: cu_q == nullptr, the
// maps cover [B, N, H, d]. Variable length: the maps cover one batch of
// total rows and Nq, Nk are the maximum lengths.
// tok_q, tok_kv: elements between consecutive tokens of q and of k/v (0 =
// contiguous: H * d and H_kv * d).
fa_status fwd_common(const void* q, const void* k, const void* v, void* out, float* lse, const int* cu_q,
                     const int* cu_k, int B, int H, int H_kv, int Nq, int Nk, int total_q, int total_k, int d,
                     fa_dtype dtype, float scale, int causal, int window_left, int window_right,
                     const float* alibi_slopes, float softcap, cudaStream_t stream, long long tok_q = 0,
                     long long tok_kv = 0) {
  const bool varlen = cu_q != nullptr;
  if (B < 0 || H < 0 || Nq < 0 || Nk < 0 || total_q < 0 || total_k < 0) return FA_ERR_SHAPE;
  if (H > 0 && (H_kv < 1 || H_kv > H || H % H_kv != 0)) return FA_ERR_SHAPE;
  if (Nq > kMaxSeq || Nk > kMaxSeq || total_q > kMaxSeq || total_k > kMaxSeq ||
      static_cast<long long>(B) * H >= (1LL << 31))
    return FA_ERR_SHAPE;
  if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_DTYPE;
  if (d != 64 && d != 128) return FA_ERR_HEADDIM;
  if (!finite(scale) || !finite(softcap) || softcap < 0.0f) return FA_ERR_ARG;
  if (window_left < -1 || window_right < -1 || (causal != 0 && causal != 1)) return FA_ERR_ARG;
  if (static_cast<long long>(B) * H * Nq == 0 || (varlen && total_q == 0)) return FA_OK;
  if (!q || !out || !lse) return FA_ERR_NULL;
  const bool any_k = varlen ? total_k > 0 : Nk > 0;
  if (any_k && (!k || !v)) return FA_ERR_NULL;
  if (!aligned16(q) || !aligned16(out) || !aligned16(k) || !aligned16(v) || !aligned16(lse)) return FA_ERR_ARG;
  const int tiles = (Nq + 127) / 128;
  if (static_cast<long long>(tiles) * B * H >= (1LL << 31)) return FA_ERR_SHAPE;
  fa_status st = check_device();
  if (st != FA_OK) return st;

  const bool bf16 = dtype == FA_BF16;
  CUtensorMap tq, tk, tv;
  // With no keys no K/V tile is ever loaded; q stands in as a valid base.
  const void* kb = any_k ? k : q;
  const void* vb = any_k ? v : q;
  const int mb = varlen ? 1 : B;
  const int nq = varlen ? total_q : Nq, nk = varlen ? total_k : Nk;
  if (!make_map(&tq, q, bf16, mb, nq, H, d, tok_q) || !make_map(&tk, kb, bf16, mb, nk, H_kv, d, tok_kv) ||
      !make_map(&tv, vb, bf16, mb, nk, H_kv, d, tok_kv))
    return FA_ERR_CUDA;

  fa::FwdParams p{};
  p.out = out;
  p.lse = lse;
  p.slopes = alibi_slopes;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.total_q = total_q;
  p.total_k = total_k;
  p.B = B;
  p.H = H;
  p.H_kv = H_kv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.num_tiles = tiles;
  p.causal = causal;
  p.window_left = window_left;
  p.window_right = window_right;
  p.use_softcap = softcap > 0.0f;
  // softmax(scale * q.k) with scale < 0 equals softmax(|scale| * (-q).k): the
  // kernel negates the QK^T product on the tensor core and works with |scale|.
  p.negate_scores = scale < 0.0f;
  const float mag = std::fabs(scale);
  p.scale_log2 = mag * fa::kLog2e;
  p.cap_scale = softcap > 0.0f ? mag / softcap : 0.0f;
  p.cap_log2 = softcap * fa::kLog2e;
  p.out_scale = 1.0f;
  return fa::launch_fwd(bf16, d, tq, tk, tv, p, stream) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

namespace {

// Backward for fixed-length (cu_q == nullptr) and packed sequences. tok: the
// token stride, in elements, of q, k, v and of dq, dk, dv when they live in
// one packed [.., 3, H, d] tensor (0 = contiguous); dout and out are always
// contiguous.
fa_status bwd_common(const void* q, const void* k, const void* v, const void* out, const float* lse,
                     const void* dout, void* dq, void* dk, void* dv, const int* cu_q, const int* cu_k, int B, int H,
                     int H_kv, int Nq, int Nk, int total_q, int total_k, int d, fa_dtype dtype, float scale,
                     int causal, int window_left, int window_right, const float* alibi_slopes, float softcap,
                     int deterministic, void* workspace, size_t workspace_bytes, cudaStream_t stream,
                     bool packed_rows = false, long long tok = 0) {
  // packed_rows: the rows are [total, H, d] (cu_q given, or B == 0 with the packed call)
  if (B < 0 || H < 1 || Nq < 0 || Nk < 0 || total_q < 0 || total_k < 0) return FA_ERR_SHAPE;
  if (H_kv < 1 || H_kv > H || H % H_kv != 0) return FA_ERR_SHAPE;
  if (Nq > kMaxSeq || Nk > kMaxSeq || total_q > kMaxSeq || total_k > kMaxSeq) return FA_ERR_SHAPE;
  // jobs of the persistent kernels (128-key blocks of every (sequence, cache
  // head); in the deterministic mode also 128-query tiles of every (sequence,
  // query head)) are numbered in an int
  if ((static_cast<long long>(Nk) + 127) / 128 * B * H_kv > INT_MAX ||
      (deterministic && (static_cast<long long>(Nq) + 127) / 128 * B * H > INT_MAX))
    return FA_ERR_SHAPE;
  if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_DTYPE;
  if (d != 64 && d != 128) return FA_ERR_HEADDIM;
  if (!finite(scale) || !finite(softcap) || softcap < 0.0f) return FA_ERR_ARG;
  if (window_left < -1 || window_right < -1 || (causal != 0 && causal != 1)) return FA_ERR_ARG;
  if (deterministic != 0 && deterministic != 1) return FA_ERR_ARG;
  // rows of q (and dq) and of k (and dk, dv)
  const long long rows_q = packed_rows ? total_q : static_cast<long long>(B) * Nq;
  const long long rows_k = packed_rows ? total_k : static_cast<long long>(B) * Nk;
  if (rows_q == 0 && rows_k == 0) return FA_OK;
  if (rows_k > 0 && (!k || !v || !dk || !dv)) return FA_ERR_NULL;
  if (rows_q > 0 && (!q || !out || !lse || !dout || !dq)) return FA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(cu_q) & 3u) || (reinterpret_cast<uintptr_t>(cu_k) & 3u))
    return FA_ERR_ARG;
  const bool work = rows_q > 0 && rows_k > 0 && Nq > 0 && Nk > 0 && B > 0;
  if (work) {
    const size_t need = fa_bwd_workspace_size(1, H, static_cast<int>(rows_q), d);
    if (!workspace || !aligned16(workspace) || workspace_bytes < need) return FA_ERR_WORKSPACE;
  }
  fa_status st = check_device();
  if (st != FA_OK) return st;
  const long long q_tok = tok > 0 ? tok : static_cast<long long>(H) * d;
  const long long kv_tok = tok > 0 ? tok : static_cast<long long>(H_kv) * d;
  if (!work) {
    // no query or no key: the gradients that exist are zero
    if (rows_k > 0 && (cudaMemset2DAsync(dk, kv_tok * 2, 0, static_cast<size_t>(H_kv) * d * 2, rows_k, stream) !=
                           cudaSuccess ||
                       cudaMemset2DAsync(dv, kv_tok * 2, 0, static_cast<size_t>(H_kv) * d * 2, rows_k, stream) !=
                           cudaSuccess))
      return FA_ERR_CUDA;
    if (rows_q > 0 &&
        cudaMemset2DAsync(dq, q_tok * 2, 0, static_cast<size_t>(H) * d * 2, rows_q, stream) != cudaSuccess)
      return FA_ERR_CUDA;
    return FA_OK;
  }
  const bool bf16 = dtype == FA_BF16;
  const int mb = packed_rows ? 1 : B, nq = packed_rows ? total_q : Nq, nk = packed_rows ? total_k : Nk;
  CUtensorMap tq, tk, tv, to, tdq;
  if (!make_map(&tq, q, bf16, mb, nq, H, d, tok, 64) || !make_map(&to, dout, bf16, mb, nq, H, d, 0, 64) ||
      !make_map(&tk, k, bf16, mb, nk, H_kv, d, tok, 64) || !make_map(&tv, v, bf16, mb, nk, H_kv, d, tok, 64) ||
      !make_map_f32(&tdq, workspace, mb, nq, H, d))
    return FA_ERR_CUDA;
  fa::BwdParams p{};
  const size_t rows = static_cast<size_t>(rows_q) * H;
  p.out = out;
  p.dout = dout;
  p.lse = lse;
  p.dq_acc = static_cast<float*>(workspace);
  p.dvec = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                    ((rows * d * sizeof(float) + 255) & ~size_t(255)));
  p.job_counter = reinterpret_cast<int*>(reinterpret_cast<char*>(p.dvec) + ((rows * sizeof(float) + 255) & ~size_t(255)));
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.dq_tok = q_tok;
  p.dkv_tok = kv_tok;
  p.slopes = alibi_slopes;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.total_q = total_q;
  p.total_k = total_k;
  p.B = B;
  p.H = H;
  p.H_kv = H_kv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.causal = causal;
  p.window_left = window_left;
  p.window_right = window_right;
  p.use_softcap = softcap > 0.0f;
  p.deterministic = deterministic;
  p.scale = scale;
  p.scale_log2 = scale * fa::kLog2e;
  p.cap_scale = softcap > 0.0f ? scale / softcap : 0.0f;
  p.cap_log2 = softcap * fa::kLog2e;
  return fa::launch_bwd(bf16, d, p, tq, tk, tv, to, tdq, stream) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status kvcache_common(const void* q, const void* k_cache, const void* v_cache, const int* block_table,
                         const int* cache_seqlens, void* out, float* lse, int B, int H, int H_kv, int d,
                         int num_pages, int page_size, int max_blocks, fa_dtype dtype, float scale,
                         int window_left, const float* alibi_slopes, float softcap, int num_splits,
                         void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (B < 0 || H < 1 || num_pages < 1 || max_blocks < 1) return FA_ERR_SHAPE;
  if (H_kv < 1 || H_kv > H || H % H_kv != 0) return FA_ERR_SHAPE;
  if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_DTYPE;
  if (d != 64 && d != 128) return FA_ERR_HEADDIM;
  if (page_size < 1 || num_splits < 0 || num_splits > FA_MAX_SPLITS) return FA_ERR_ARG;
  if (!finite(scale) || !finite(softcap) || softcap < 0.0f || window_left < -1) return FA_ERR_ARG;
  if (!kvcache_sizes_ok(B, H, d, max_blocks, page_size)) return FA_ERR_SHAPE;
  if (B == 0) return FA_OK;
  if (!q || !k_cache || !v_cache || !block_table || !cache_seqlens || !out || !lse) return FA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out)) return FA_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(cache_seqlens) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_ARG;
  const int S = launch_splits(B, H, H_kv, d, max_blocks, page_size, num_splits);
  if (S < 1) return FA_ERR_SHAPE;
  if (S > 1 && (!workspace || !aligned16(workspace) || workspace_bytes < partial_bytes(S, B, H, d)))
    return FA_ERR_WORKSPACE;
  fa_status st = check_device();
  if (st != FA_OK) return st;

  fa::DecodeParams p{};
  p.q = q;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.block_table = block_table;
  p.cache_seqlens = cache_seqlens;
  p.out = out;
  p.lse = lse;
  if (S > 1) {
    const size_t rows = static_cast<size_t>(S) * B * H;
    p.o_part = static_cast<float*>(workspace);
    p.lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + partial_bytes(S, B, H, d) -
                                          rows * sizeof(float));
  }
  p.slopes = alibi_slopes;
  p.B = B;
  p.H = H;
  p.H_kv = H_kv;
  p.num_pages = num_pages;
  p.page_size = page_size;
  p.max_blocks = max_blocks;
  p.num_splits = S;
  p.window_left = window_left;
  p.use_softcap = softcap > 0.0f;
  p.scale_log2 = scale * fa::kLog2e;
  p.cap_scale = softcap > 0.0f ? scale / softcap : 0.0f;
  p.cap_log2 = softcap * fa::kLog2e;
  const bool bf16 = dtype == FA_BF16;
  if (page_size % 64 == 0) {
    CUtensorMap tk, tv;
    const bool sw = fa::decode_on_tensor_cores(H, H_kv);
    if (!make_cache_map(&tk, k_cache, bf16, num_pages, page_size, H_kv, d, sw) ||
        !make_cache_map(&tv, v_cache, bf16, num_pages, page_size, H_kv, d, sw))
      return FA_ERR_CUDA;
    return fa::launch_decode(bf16, d, p, &tk, &tv, stream) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
  }
  return fa::launch_decode(bf16, d, p, nullptr, nullptr, stream) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_NULL: return "FA_ERR_NULL: a required pointer is NULL";
    case FA_ERR_SHAPE: return "FA_ERR_SHAPE: a size is out of range";
    case FA_ERR_DTYPE: return "FA_ERR_DTYPE: dtype must be FA_FP16 or FA_BF16";
    case FA_ERR_HEADDIM: return "FA_ERR_HEADDIM: head dimension must be 64 or 128";
    case FA_ERR_ARG: return "FA_ERR_ARG: invalid scalar argument or unaligned pointer";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE: split-KV workspace missing, misaligned or too small";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: a CUDA call or kernel launch failed";
    case FA_ERR_DEVICE: return "FA_ERR_DEVICE: no CUDA device or the device is not sm_100";
  }
  return "unknown fa_status";
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H, int Nq, int Nk,
                 int d, fa_dtype dtype, float scale, int causal, int window_left, int window_right,
                 const float* alibi_slopes, float softcap, cudaStream_t stream) {
  return fwd_common(q, k, v, out, lse, nullptr, nullptr, B, H, H, Nq, Nk, 0, 0, d, dtype, scale, causal,
                    window_left, window_right, alibi_slopes, softcap, stream);
}

fa_status fa_fwd_gqa(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H, int H_kv,
                     int Nq, int Nk, int d, fa_dtype dtype, float scale, int causal, int window_left,
                     int window_right, const float* alibi_slopes, float softcap, cudaStream_t stream) {
  return fwd_common(q, k, v, out, lse, nullptr, nullptr, B, H, H_kv, Nq, Nk, 0, 0, d, dtype, scale, causal,
                    window_left, window_right, alibi_slopes, softcap, stream);
}

fa_status fa_fwd_qkvpacked(const void* qkv, void* out, float* lse, int B, int H, int N, int d, fa_dtype dtype,
                           float scale, int causal, int window_left, int window_right, const float* alibi_slopes,
                           float softcap, cudaStream_t stream) {
  const long long hd = static_cast<long long>(H) * d;
  const char* base = static_cast<const char*>(qkv);
  const void* k = base ? base + hd * 2 : nullptr;
  const void* v = base ? base + 2 * hd * 2 : nullptr;
  return fwd_common(qkv, k, v, out, lse, nullptr, nullptr, B, H, H, N, N, 0, 0, d, dtype, scale, causal,
                    window_left, window_right, alibi_slopes, softcap, stream, 3 * hd, 3 * hd);
}

fa_status fa_fwd_varlen_qkvpacked(const void* qkv, void* out, float* lse, const int* cu_seqlens, int B, int H,
                                  int max_seqlen, int total, int d, fa_dtype dtype, float scale, int causal,
                                  int window_left, int window_right, const float* alibi_slopes, float softcap,
                                  cudaStream_t stream) {
  if (B > 0 && !cu_seqlens) return FA_ERR_NULL;
  const long long hd = static_cast<long long>(H) * d;
  const char* base = static_cast<const char*>(qkv);
  const void* k = base ? base + hd * 2 : nullptr;
  const void* v = base ? base + 2 * hd * 2 : nullptr;
  return fwd_common(qkv, k, v, out, lse, cu_seqlens, cu_seqlens, B, H, H, max_seqlen, max_seqlen, total, total, d,
                    dtype, scale, causal, window_left, window_right, alibi_slopes, softcap, stream, 3 * hd, 3 * hd);
}

fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* out, float* lse,
                        const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int H, int max_seqlen_q,
                        int max_seqlen_k, int total_q, int total_k, int d, fa_dtype dtype, float scale, int causal,
                        int window_left, int window_right, const float* alibi_slopes, float softcap,
                        cudaStream_t stream) {
  if (B > 0 && (!cu_seqlens_q || !cu_seqlens_k)) return FA_ERR_NULL;
  return fwd_common(q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k, B, H, H, max_seqlen_q, max_seqlen_k, total_q,
                    total_k, d, dtype, scale, causal, window_left, window_right, alibi_slopes, softcap, stream);
}

int fa_kvcache_num_splits(int B, int H, int d, int max_blocks, int page_size, int num_splits) {
  if (!kvcache_sizes_ok(B, H, d, max_blocks, page_size)) return -1;
  if (num_splits < 0 || num_splits > FA_MAX_SPLITS) return -1;
  if (num_splits > 0) return num_splits;
  if (B == 0) return 1;
  return auto_splits(B, H, static_cast<long long>(max_blocks) * page_size);
}

size_t fa_fwd_fp8_workspace_size(int B, int H_kv, int Nk, int d) {
  if (B < 0 || H_kv < 1 || Nk < 0 || d != 128 || Nk > kMaxSeq) return 0;
  return static_cast<size_t>(B) * H_kv * d * static_cast<size_t>(fp8_keys_padded(Nk));
}

fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H, int H_kv,
                     int Nq, int Nk, int d, fa_fp8_format fmt, float scale, float descale_q, float descale_k,
                     float descale_v, int causal, int window_left, int window_right, const float* alibi_slopes,
                     float softcap, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (B < 0 || H < 0 || Nq < 0 || Nk < 0) return FA_ERR_SHAPE;
  if (H > 0 && (H_kv < 1 || H_kv > H || H % H_kv != 0)) return FA_ERR_SHAPE;
  if (Nq > kMaxSeq || Nk > kMaxSeq || static_cast<long long>(B) * H >= (1LL << 31)) return FA_ERR_SHAPE;
  if (B > 65535 || H_kv > 65535) return FA_ERR_SHAPE;  // grid of the V transpose
  if (fmt != FA_E4M3 && fmt != FA_E5M2) return FA_ERR_DTYPE;
  if (d != 128) return FA_ERR_HEADDIM;
  if (!finite(scale) || !finite(softcap) || softcap < 0.0f) return FA_ERR_ARG;
  if (!finite(descale_q) || !finite(descale_k) || !finite(descale_v) || descale_q <= 0.0f || descale_k <= 0.0f ||
      descale_v <= 0.0f)
    return FA_ERR_ARG;
  if (window_left < -1 || window_right < -1 || (causal != 0 && causal != 1)) return FA_ERR_ARG;
  if (static_cast<long long>(B) * H * Nq == 0) return FA_OK;
  if (!q || !out || !lse) return FA_ERR_NULL;
  if (Nk > 0 && (!k || !v)) return FA_ERR_NULL;
  if (!aligned16(q) || !aligned16(out) || !aligned16(k) || !aligned16(v) || !aligned16(lse)) return FA_ERR_ARG;
  const int tiles = (Nq + 127) / 128;
  if (static_cast<long long>(tiles) * B * H >= (1LL << 31)) return FA_ERR_SHAPE;
  const size_t need = fa_fwd_fp8_workspace_size(B, H_kv, Nk, d);
  if (need > 0 && (!workspace || !aligned16(workspace) || workspace_bytes < need)) return FA_ERR_WORKSPACE;
  fa_status st = check_device();
  if (st != FA_OK) return st;

  const int Nk_pad = static_cast<int>(fp8_keys_padded(Nk));
  CUtensorMap tq, tk, tvt;
  // with no keys no K or V tile is ever loaded; q stands in as a valid base
  const void* kb = Nk > 0 ? k : q;
  void* vtb = Nk > 0 ? workspace : const_cast<void*>(q);
  if (!make_map_u8(&tq, q, B, Nq, H, d) || !make_map_u8(&tk, kb, B, Nk, H_kv, d) ||
      !make_map_vt(&tvt, vtb, B, H_kv, d, Nk > 0 ? Nk_pad : 16))
    return FA_ERR_CUDA;
  if (Nk > 0 && fa::launch_v_transpose(v, workspace, B, Nk, H_kv, Nk_pad, stream) != cudaSuccess) return FA_ERR_CUDA;

  fa::FwdParams p{};
  p.out = out;
  p.lse = lse;
  p.slopes = alibi_slopes;
  p.B = B;
  p.H = H;
  p.H_kv = H_kv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.num_tiles = tiles;
  p.causal = causal;
  p.window_left = window_left;
  p.window_right = window_right;
  p.use_softcap = softcap > 0.0f;
  // the scores of the 8-bit values are scaled by scale * descale_q *
  // descale_k; O by descale_v
  const float eff = scale * descale_q * descale_k;
  if (!finite(eff)) return FA_ERR_ARG;
  p.negate_scores = eff < 0.0f;
  const float mag = std::fabs(eff);
  p.scale_log2 = mag * fa::kLog2e;
  p.cap_scale = softcap > 0.0f ? mag / softcap : 0.0f;
  p.cap_log2 = softcap * fa::kLog2e;
  p.out_scale = descale_v;
  return fa::launch_fwd_fp8(fmt == FA_E5M2 ? 1 : 0, tq, tk, tvt, p, stream) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_kvcache_num_splits_gqa(int B, int H, int H_kv, int d, int max_blocks, int page_size, int num_splits) {
  return launch_splits(B, H, H_kv, d, max_blocks, page_size, num_splits);
}

size_t fa_kvcache_workspace_size(int B, int H, int d, int max_blocks, int page_size, int num_splits) {
  const int s = fa_kvcache_num_splits(B, H, d, max_blocks, page_size, num_splits);
  return s > 1 ? partial_bytes(s, B, H, d) : 0;
}

fa_status fa_fwd_kvcache(const void* q, const void* k_cache, const void* v_cache, const int* block_table,
                         const int* cache_seqlens, void* out, float* lse, int B, int H, int d, int num_pages,
                         int page_size, int max_blocks, fa_dtype dtype, float scale, int window_left,
                         const float* alibi_slopes, float softcap, int num_splits, void* workspace,
                         size_t workspace_bytes, cudaStream_t stream) {
  return kvcache_common(q, k_cache, v_cache, block_table, cache_seqlens, out, lse, B, H, H, d, num_pages, page_size,
                        max_blocks, dtype, scale, window_left, alibi_slopes, softcap, num_splits, workspace,
                        workspace_bytes, stream);
}

fa_status fa_fwd_kvcache_gqa(const void* q, const void* k_cache, const void* v_cache, const int* block_table,
                             const int* cache_seqlens, void* out, float* lse, int B, int H, int H_kv, int d,
                             int num_pages, int page_size, int max_blocks, fa_dtype dtype, float scale,
                             int window_left, const float* alibi_slopes, float softcap, int num_splits,
                             void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return kvcache_common(q, k_cache, v_cache, block_table, cache_seqlens, out, lse, B, H, H_kv, d, num_pages,
                        page_size, max_blocks, dtype, scale, window_left, alibi_slopes, softcap, num_splits,
                        workspace, workspace_bytes, stream);
}

fa_status fa_kvcache_append(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                            const int* block_table, const int* cache_seqlens, int B, int n_new, int H_kv, int d,
                            int num_pages, int page_size, int max_blocks, fa_dtype dtype, cudaStream_t stream) {
  if (B < 0 || n_new < 0 || H_kv < 1 || num_pages < 1 || max_blocks < 1) return FA_ERR_SHAPE;
  if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_DTYPE;
  if (d != 64 && d != 128) return FA_ERR_HEADDIM;
  if (page_size < 1) return FA_ERR_ARG;
  if (static_cast<long long>(max_blocks) * page_size >= (1LL << 31) ||
      static_cast<long long>(B) * n_new * H_kv >= (1LL << 31) || B > 65535)
    return FA_ERR_SHAPE;
  if (static_cast<long long>(B) * n_new == 0) return FA_OK;
  if (!k_new || !v_new || !k_cache || !v_cache || !block_table || !cache_seqlens) return FA_ERR_NULL;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache)) return FA_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(cache_seqlens) & 3u))
    return FA_ERR_ARG;
  fa_status st = check_device();
  if (st != FA_OK) return st;
  fa::AppendParams p{};
  p.k_new = k_new;
  p.v_new = v_new;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.block_table = block_table;
  p.cache_seqlens = cache_seqlens;
  p.B = B;
  p.n_new = n_new;
  p.H_kv = H_kv;
  p.d = d;
  p.num_pages = num_pages;
  p.page_size = page_size;
  p.max_blocks = max_blocks;
  return fa::launch_append(p, stream) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_bwd_workspace_size(int B, int H, int Nq, int d) {
  if (B < 0 || H < 0 || Nq < 0 || d < 0) return 0;
  const size_t rows = static_cast<size_t>(B) * H * Nq;
  // fp32 dQ accumulator, D, and the job counter of the tensor-core kernel
  return ((rows * d * sizeof(float) + 255) & ~size_t(255)) + ((rows * sizeof(float) + 255) & ~size_t(255)) + 256;
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
                 void* dq, void* dk, void* dv, int B, int H, int H_kv, int Nq, int Nk, int d, fa_dtype dtype,
                 float scale, int causal, int window_left, int window_right, const float* alibi_slopes,
                 float softcap, int deterministic, void* workspace, size_t workspace_bytes,
                 cudaStream_t stream) {
  return bwd_common(q, k, v, out, lse, dout, dq, dk, dv, nullptr, nullptr, B, H, H_kv, Nq, Nk, 0, 0, d, dtype, scale,
                    causal, window_left, window_right, alibi_slopes, softcap, deterministic, workspace,
                    workspace_bytes, stream);
}

fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* out, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, const int* cu_seqlens_q,
                        const int* cu_seqlens_k, int B, int H, int H_kv, int max_seqlen_q, int max_seqlen_k,
                        int total_q, int total_k, int d, fa_dtype dtype, float scale, int causal, int window_left,
                        int window_right, const float* alibi_slopes, float softcap, int deterministic,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (B > 0 && (!cu_seqlens_q || !cu_seqlens_k)) return FA_ERR_NULL;
  if (B < 0) return FA_ERR_SHAPE;
  return bwd_common(q, k, v, out, lse, dout, dq, dk, dv, B > 0 ? cu_seqlens_q : nullptr,
                    B > 0 ? cu_seqlens_k : nullptr, B, H, H_kv, max_seqlen_q, max_seqlen_k, total_q, total_k, d,
                    dtype, scale, causal, window_left, window_right, alibi_slopes, softcap, deterministic, workspace,
                    workspace_bytes, stream, true);
}

fa_status fa_bwd_qkvpacked(const void* qkv, const void* out, const float* lse, const void* dout, void* dqkv, int B,
                           int H, int N, int d, fa_dtype dtype, float scale, int causal, int window_left,
                           int window_right, const float* alibi_slopes, float softcap, int deterministic,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const long long hd = static_cast<long long>(H) * d;
  const char* in = static_cast<const char*>(qkv);
  char* o = static_cast<char*>(dqkv);
  return bwd_common(qkv, in ? in + hd * 2 : nullptr, in ? in + 2 * hd * 2 : nullptr, out, lse, dout, dqkv,
                    o ? o + hd * 2 : nullptr, o ? o + 2 * hd * 2 : nullptr, nullptr, nullptr, B, H, H, N, N, 0, 0, d,
                    dtype, scale, causal, window_left, window_right, alibi_slopes, softcap, deterministic, workspace,
                    workspace_bytes, stream, false, 3 * hd);
}

fa_status fa_bwd_varlen_qkvpacked(const void* qkv, const void* out, const float* lse, const void* dout, void* dqkv,
                                  const int* cu_seqlens, int B, int H, int max_seqlen, int total, int d,
                                  fa_dtype dtype, float scale, int causal, int window_left, int window_right,
                                  const float* alibi_slopes, float softcap, int deterministic, void* workspace,
                                  size_t workspace_bytes, cudaStream_t stream) {
  if (B > 0 && !cu_seqlens) return FA_ERR_NULL;
  if (B < 0) return FA_ERR_SHAPE;
  const long long hd = static_cast<long long>(H) * d;
  const char* in = static_cast<const char*>(qkv);
  char* o = static_cast<char*>(dqkv);
  return bwd_common(qkv, in ? in + hd * 2 : nullptr, in ? in + 2 * hd * 2 : nullptr, out, lse, dout, dqkv,
                    o ? o + hd * 2 : nullptr, o ? o + 2 * hd * 2 : nullptr, B > 0 ? cu_seqlens : nullptr,
                    B > 0 ? cu_seqlens : nullptr, B, H, H, max_seqlen, max_seqlen, total, total, d, dtype, scale,
                    causal, window_left, window_right, alibi_slopes, softcap, deterministic, workspace,
                    workspace_bytes, stream, true, 3 * hd);
}

}  // extern "C"
